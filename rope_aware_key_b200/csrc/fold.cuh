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
// fp64 throughout (w_f * delta reaches 2^16 rad for the default schedule, far
// beyond what fp32 phases can hold); fp32 output.
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

// The averaged fold.  The offset mean and the kept distance depend only on
// (theta, D, delta0), so the host sums them in fp64 into one complex factor
// per band, A_f = W_f e^{i w_f delta0}; the kernel maps every center:
// a_f = E[q_f] A_f (fp64), stored as fp32.
struct FoldArgs {
  const float* q;     // [n_centers][128]
  float* w;           // [n_centers][128]
  int n_centers;
  int pairing;
  double a_re[kBands], a_im[kBands];
};

__global__ void __launch_bounds__(kThreads) fold_kernel(const __grid_constant__ FoldArgs a) {
  const int ci = blockIdx.x * kThreads + threadIdx.x;
  if (ci >= a.n_centers * kBands) return;
  const int c = ci / kBands, f = ci - c * kBands;
  const int re = a.pairing == TRI_PAIRING_HALF ? f : 2 * f;
  const int im = a.pairing == TRI_PAIRING_HALF ? f + kBands : 2 * f + 1;
  const float* q = a.q + static_cast<int64_t>(c) * kD;
  const float qr_f = q[re], qi_f = q[im];
  if (!isfinite(qr_f) || !isfinite(qi_f)) flag(TRI_DEVFLAG_NONFINITE);
  const double qr = qr_f, qi = qi_f;
  const double ar = a.a_re[f], ai = a.a_im[f];
  float* w = a.w + static_cast<int64_t>(c) * kD;
  w[re] = static_cast<float>(ar * qr - ai * qi);
  w[im] = static_cast<float>(ai * qr + ar * qi);
}

// Per-offset weights for the max-over-offsets score (no averaging):
//   a_{f,t} = E[q_f] e^{i w_f (delta0 + delta_t)},  w[c][t][re(f)] = Re, w[c][t][im(f)] = Im.
// The rotation depends only on (band, offset): a block takes one offset and
// kFoldCenters centers, a thread one band and kFoldPer of those centers, so
// each thread evaluates its rotation once (fp64 sincos) and applies it to its
// centers (fp64 products, fp32 out), their loads issued together; loads and
// stores of a center's bands are contiguous across the threads.
constexpr int kFoldCenters = 32;                   // centers per block
constexpr int kFoldRows = 4;                       // threads per band
constexpr int kFoldPer = kFoldCenters / kFoldRows; // centers per thread

template <int N>
__global__ void __launch_bounds__(kBands * kFoldRows) fold_offsets_kernel(const __grid_constant__ Args<N> a) {
  const int f = threadIdx.x, t = blockIdx.x;
  if (t == 0 && blockIdx.y == 0 && f == 0 && threadIdx.y == 0) {
    bool finite = isfinite(a.theta) && isfinite(a.delta0);
    for (int o = 0; o < a.n_offsets; ++o) finite = finite && isfinite(a.offsets[o]);
    if (!finite) flag(TRI_DEVFLAG_NONFINITE);
  }
  const int re = a.pairing == TRI_PAIRING_HALF ? f : 2 * f;
  const int im = a.pairing == TRI_PAIRING_HALF ? f + kBands : 2 * f + 1;
  const int cb = blockIdx.y * kFoldCenters + threadIdx.y;
  float qr[kFoldPer], qi[kFoldPer];
#pragma unroll
  for (int i = 0; i < kFoldPer; ++i) {
    const int c = cb + i * kFoldRows;
    const float* q = a.q + static_cast<int64_t>(c < a.n_centers ? c : 0) * kD;
    qr[i] = q[re];
    qi[i] = q[im];
  }
  double sn, cs;
  sincos(a.omega[f] * (a.delta0 + a.offsets[t]), &sn, &cs);
#pragma unroll
  for (int i = 0; i < kFoldPer; ++i) {
    const int c = cb + i * kFoldRows;
    if (c >= a.n_centers) break;
    if (!isfinite(qr[i]) || !isfinite(qi[i])) flag(TRI_DEVFLAG_NONFINITE);
    const double dr = qr[i], di = qi[i];
    float* w = a.w + (static_cast<int64_t>(c) * a.n_offsets + t) * kD;
    w[re] = static_cast<float>(cs * dr - sn * di);
    w[im] = static_cast<float>(sn * dr + cs * di);
  }
}

}  // namespace fold
}  // namespace tri
