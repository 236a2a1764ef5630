// Offline fold of the offset average into one real weight vector per center.
//
// Page "The future-offset average in TriAttention can be precomputed",
// section "The averaging step - the one we improve": because
// e^{i w (Delta + delta)} = e^{i w Delta} e^{i w delta}, the average over the
// schedule D reaches only the offset factor and collapses into
//     W_f = (1/|D|) sum_{delta in D} e^{i w_f delta},
// and the averaged score is one evaluation with the center replaced by
// mu'_f = E[q_f] W_f.  The closing remark of the section folds this into the
// real coefficients as a fixed 2x2 map per band; with the kept distance
// delta0 folded in as well,
//     a_f = E[q_f] W_f e^{i w_f delta0},   w[re(f)] = Re a_f,  w[im(f)] = Im a_f,
// and Re sum_f a_f conj(k_f) = sum_j w[j] k[j].
//
// Grid: one CTA per (band f, block of kThreads centers).  Each CTA sums W_f
// over the schedule with a fixed-order fp64 tree, then maps its centers'
// band f.  fp64 throughout (w_f * delta reaches 2^16 rad for the default
// schedule, far beyond what fp32 phases can hold); fp32 output.
#pragma once

#include "common.cuh"

namespace tri {
namespace fold {

constexpr int kThreads = 256;
constexpr int kBands = kD / 2;

// The schedule travels in the kernel parameters; short schedules (the usual
// case) use a small parameter block, which launches faster than the largest.
constexpr int kSmallOffsets = 64;

template <int MAX_OFFSETS>
struct Args {
  const float* q;     // [n_centers][128]
  float* w;           // [n_centers][128]
  int n_centers;
  int pairing;
  double theta;
  double delta0;
  int n_offsets;
  double omega[kBands];            // theta^(-2f/128), computed on the host in fp64
  double offsets[MAX_OFFSETS];
};

template <int N>
__global__ void __launch_bounds__(kThreads) fold_kernel(const __grid_constant__ Args<N> a) {
  __shared__ double s_c[kThreads / 32], s_s[kThreads / 32];
  const int f = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const double omega = a.omega[f];

  // W_f = mean over the schedule of e^{i omega delta}
  double c = 0.0, s = 0.0;
  for (int t = threadIdx.x; t < a.n_offsets; t += kThreads) {
    double sn, cs;
    sincos(omega * a.offsets[t], &sn, &cs);
    c += cs;
    s += sn;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    s += __shfl_xor_sync(0xffffffffu, s, o);
  }
  if (lane == 0) {
    s_c[warp] = c;
    s_s[warp] = s;
  }
  __syncthreads();
  double wre = 0.0, wim = 0.0;
  for (int i = 0; i < kThreads / 32; ++i) {
    wre += s_c[i];
    wim += s_s[i];
  }
  wre /= a.n_offsets;
  wim /= a.n_offsets;

  if (f == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    bool finite = isfinite(a.theta) && isfinite(a.delta0);
    for (int t = 0; t < a.n_offsets; ++t) finite = finite && isfinite(a.offsets[t]);
    if (!finite) flag(TRI_DEVFLAG_NONFINITE);
  }

  const int ci = blockIdx.y * kThreads + threadIdx.x;
  if (ci >= a.n_centers) return;
  const int re = a.pairing == TRI_PAIRING_HALF ? f : 2 * f;
  const int im = a.pairing == TRI_PAIRING_HALF ? f + kBands : 2 * f + 1;
  const float* q = a.q + static_cast<int64_t>(ci) * kD;
  const float qr_f = q[re], qi_f = q[im];
  if (!isfinite(qr_f) || !isfinite(qi_f)) flag(TRI_DEVFLAG_NONFINITE);
  const double qr = qr_f, qi = qi_f;
  // mu'_f = E[q_f] W_f
  const double mr = wre * qr - wim * qi;
  const double mi = wim * qr + wre * qi;
  double ar = mr, ai = mi;
  if (a.delta0 != 0.0) {
    double sn, cs;
    sincos(omega * a.delta0, &sn, &cs);
    ar = cs * mr - sn * mi;
    ai = sn * mr + cs * mi;
  }
  float* w = a.w + static_cast<int64_t>(ci) * kD;
  w[re] = static_cast<float>(ar);
  w[im] = static_cast<float>(ai);
}

// Per-offset weights for the max-over-offsets score (no averaging):
//   a_{f,t} = E[q_f] e^{i w_f (delta0 + delta_t)},  w[c][t][re(f)] = Re, w[c][t][im(f)] = Im.
// Grid: (band f, block of kThreads (center, offset) pairs); fp64, fp32 out.
template <int N>
__global__ void __launch_bounds__(kThreads) fold_offsets_kernel(const __grid_constant__ Args<N> a) {
  const int f = blockIdx.x;
  const double omega = a.omega[f];
  if (f == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    bool finite = isfinite(a.theta) && isfinite(a.delta0);
    for (int t = 0; t < a.n_offsets; ++t) finite = finite && isfinite(a.offsets[t]);
    if (!finite) flag(TRI_DEVFLAG_NONFINITE);
  }
  const int idx = blockIdx.y * kThreads + threadIdx.x;
  if (idx >= a.n_centers * a.n_offsets) return;
  const int c = idx / a.n_offsets, t = idx - c * a.n_offsets;
  const int re = a.pairing == TRI_PAIRING_HALF ? f : 2 * f;
  const int im = a.pairing == TRI_PAIRING_HALF ? f + kBands : 2 * f + 1;
  const float* q = a.q + static_cast<int64_t>(c) * kD;
  const float qr_f = q[re], qi_f = q[im];
  if (!isfinite(qr_f) || !isfinite(qi_f)) flag(TRI_DEVFLAG_NONFINITE);
  double sn, cs;
  sincos(omega * (a.delta0 + a.offsets[t]), &sn, &cs);
  const double qr = qr_f, qi = qi_f;
  float* w = a.w + static_cast<int64_t>(idx) * kD;
  w[re] = static_cast<float>(cs * qr - sn * qi);
  w[im] = static_cast<float>(sn * qr + cs * qi);
}

}  // namespace fold
}  // namespace tri
