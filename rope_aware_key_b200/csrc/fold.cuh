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
// One CTA; fp64 throughout (w_f * delta reaches 2^16 rad for the default
// schedule, far beyond what fp32 phases can hold), fp32 output.
#pragma once

#include "common.cuh"

namespace tri {
namespace fold {

constexpr int kThreads = 512;
constexpr int kBands = kD / 2;

struct Args {
  const float* q;     // [n_centers][128]
  float* w;           // [n_centers][128]
  int n_centers;
  int pairing;
  double theta;
  double delta0;
  int n_offsets;
  double offsets[TRI_MAX_OFFSETS];
};

__global__ void __launch_bounds__(kThreads) fold_kernel(const __grid_constant__ Args a) {
  __shared__ double s_wre[kBands], s_wim[kBands], s_omega[kBands];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kThreads / 32;

  // W_f: warp-per-band sums over the schedule, fixed reduction order.
  for (int f = warp; f < kBands; f += kWarps) {
    const double omega = pow(a.theta, -2.0 * f / kD);
    double c = 0.0, s = 0.0;
    for (int t = lane; t < a.n_offsets; t += 32) {
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
      s_wre[f] = c / a.n_offsets;
      s_wim[f] = s / a.n_offsets;
      s_omega[f] = omega;
    }
  }
  if (threadIdx.x == 0) {
    bool finite = isfinite(a.theta) && isfinite(a.delta0);
    for (int t = 0; t < a.n_offsets; ++t) finite = finite && isfinite(a.offsets[t]);
    if (!finite) flag(TRI_DEVFLAG_NONFINITE);
  }
  __syncthreads();

  // a_f for every (center, band).
  const int total = a.n_centers * kBands;
  for (int idx = threadIdx.x; idx < total; idx += kThreads) {
    const int c = idx / kBands, f = idx - c * kBands;
    const int re = a.pairing == TRI_PAIRING_HALF ? f : 2 * f;
    const int im = a.pairing == TRI_PAIRING_HALF ? f + kBands : 2 * f + 1;
    const float* q = a.q + static_cast<int64_t>(c) * kD;
    const float qr_f = q[re], qi_f = q[im];
    if (!isfinite(qr_f) || !isfinite(qi_f)) flag(TRI_DEVFLAG_NONFINITE);
    const double qr = qr_f, qi = qi_f;
    // mu' = E[q_f] W_f
    const double mr = s_wre[f] * qr - s_wim[f] * qi;
    const double mi = s_wim[f] * qr + s_wre[f] * qi;
    double ar = mr, ai = mi;
    if (a.delta0 != 0.0) {
      double sn, cs;
      sincos(s_omega[f] * a.delta0, &sn, &cs);
      ar = cs * mr - sn * mi;
      ai = sn * mr + cs * mi;
    }
    float* w = a.w + static_cast<int64_t>(c) * kD;
    w[re] = static_cast<float>(ar);
    w[im] = static_cast<float>(ai);
  }
}

}  // namespace fold
}  // namespace tri
