// Keep-highest selection: per unit, the top min(B, n) keys under the order
// (score descending, index ascending), written as ascending indices.
//
// Page "The future-offset average in TriAttention can be precomputed",
// opening section: the cache keeps its highest-scoring keys within a memory
// budget.  The budget B is TriAttention's KV budget (README, default 2048).
//
// One CTA per unit, on the unit's row of the score matrix (L2-resident right
// after scoring):
//  1. map each fp32 score to an order-preserving uint32 key (NaN -> 0, the
//     lowest; -0 -> +0);
//  2. min/max of the keys; their common leading bits are shared by every key,
//     so the radix search starts below them;
//  3. radix select, 11 bits per pass, with a shared-memory histogram of the
//     keys that still match the prefix found so far: gives the threshold T
//     (the B-th largest key) and `need`, how many keys equal to T are kept;
//  4. one ordered pass: key i is kept iff key > T, or key == T and fewer than
//     `need` keys equal to T precede it.  Its output slot is the number of kept
//     keys before it (a block-wide exclusive scan of (greater, equal) counts),
//     so the output is ascending and the result never depends on the order of
//     atomics.
#pragma once

#include "common.cuh"

namespace tri {
namespace select {

constexpr int kDigitBits = 11;
constexpr int kBins = 1 << kDigitBits;

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (s != s) return 0u;               // NaN ranks lowest
  if (u == 0x80000000u) u = 0u;        // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Args {
  const float* scores;
  int32_t* kept;
  int32_t* kept_count;
  int B;
};

// Visit the keys of one row: fn(i, key) for i in [0, n), 4 per thread per
// step (16-byte loads; the row start is 16-byte aligned).
template <int NT, typename Fn>
__device__ __forceinline__ void for_each_key(const float* __restrict__ row, int n, Fn fn) {
  for (int base = threadIdx.x * 4; base < n; base += NT * 4) {
    if (base + 3 < n) {
      const float4 v = *reinterpret_cast<const float4*>(row + base);
      fn(base + 0, order_key(v.x));
      fn(base + 1, order_key(v.y));
      fn(base + 2, order_key(v.z));
      fn(base + 3, order_key(v.w));
    } else {
      for (int i = base; i < n; ++i) fn(i, order_key(row[i]));
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(const __grid_constant__ Geom g, const Args a) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t scan_sh[NT / 32];
  __shared__ uint32_t red_min[NT / 32], red_max[NT / 32];
  __shared__ uint32_t s_digit, s_above;

  const int u = blockIdx.x;
  const int b = u % g.batch;
  const int n = g.len[b];
  const int B = a.B;
  const float* __restrict__ row = a.scores + static_cast<int64_t>(u) * g.score_stride;
  int32_t* __restrict__ kept = a.kept + static_cast<int64_t>(u) * B;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) a.kept_count[u] = min(n, B);
  if (n <= B) {
    for (int i = threadIdx.x; i < n; i += NT) kept[i] = i;
    return;
  }

  // ---- min / max of the keys
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for_each_key<NT>(row, n, [&](int, uint32_t key) {
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  });
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    red_min[warp] = kmin;
    red_max[warp] = kmax;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < NT / 32 ? red_min[lane] : 0xffffffffu;
    uint32_t y = lane < NT / 32 ? red_max[lane] : 0u;
    x = __reduce_min_sync(0xffffffffu, x);
    y = __reduce_max_sync(0xffffffffu, y);
    if (lane == 0) {
      red_min[0] = x;
      red_max[0] = y;
    }
  }
  __syncthreads();
  kmin = red_min[0];
  kmax = red_max[0];

  // ---- radix search for the threshold
  uint32_t prefix;
  uint32_t need = static_cast<uint32_t>(B);     // still to take among keys matching prefix
  if (kmin == kmax) {
    prefix = kmax;
  } else {
    int known = __clz(kmin ^ kmax);             // leading bits common to every key
    prefix = known ? (kmax & (0xffffffffu << (32 - known))) : 0u;
    while (known < 32) {
      const int bits = min(kDigitBits, 32 - known);
      const int shift = 32 - known - bits;
      const int nbins = 1 << bits;
      for (int i = threadIdx.x; i < nbins; i += NT) hist[i] = 0;
      __syncthreads();
      const uint32_t pfx = prefix;
      const int kn = known;
      for_each_key<NT>(row, n, [&](int, uint32_t key) {
        const bool match = kn == 0 || ((key ^ pfx) >> (32 - kn)) == 0u;
        if (match) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
      });
      __syncthreads();
      if (warp == 0) {
        // lane 0 owns the top chunk of bins, lane 31 the bottom one
        const int chunk = (nbins + 31) / 32;
        const int hi = nbins - lane * chunk;
        const int lo = max(0, hi - chunk);
        uint32_t sum = 0;
        for (int i = lo; i < hi; ++i) sum += hist[i];
        uint32_t cum = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, cum, o);
          if (lane >= o) cum += y;
        }
        const uint32_t ballot = __ballot_sync(0xffffffffu, cum >= need);
        const int owner = __ffs(ballot) - 1;
        if (lane == owner) {
          uint32_t above = cum - sum;
          int d = lo;
          for (int i = hi - 1; i >= lo; --i) {
            if (above + hist[i] >= need) {
              d = i;
              break;
            }
            above += hist[i];
          }
          s_digit = static_cast<uint32_t>(d);
          s_above = above;
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      need -= s_above;
      known += bits;
      __syncthreads();   // hist and s_digit are rewritten in the next pass
    }
  }
  const uint32_t T = prefix;

  // ---- ordered emit
  uint32_t run_gt = 0, run_eq = 0;     // counts over all earlier chunks
  for (int base = 0; base < n; base += NT * 4) {
    const int i0 = base + threadIdx.x * 4;
    uint32_t key[4];
    if (i0 + 3 < n) {
      const float4 v = *reinterpret_cast<const float4*>(row + i0);
      key[0] = order_key(v.x);
      key[1] = order_key(v.y);
      key[2] = order_key(v.z);
      key[3] = order_key(v.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) key[e] = i0 + e < n ? order_key(row[i0 + e]) : 0u;
    }
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = i0 + e < n;
      gt += (valid && key[e] > T);
      eq += (valid && key[e] == T);
    }
    uint32_t total;
    const uint32_t pre = block_exclusive_sum<NT>((gt << 16) | eq, scan_sh, &total);
    uint32_t gt_before = run_gt + (pre >> 16);
    uint32_t eq_before = run_eq + (pre & 0xffffu);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i0 + e >= n) break;
      if (key[e] > T) {
        kept[gt_before + min(eq_before, need)] = i0 + e;
        ++gt_before;
      } else if (key[e] == T) {
        if (eq_before < need) kept[gt_before + eq_before] = i0 + e;
        ++eq_before;
      }
    }
    run_gt += total >> 16;
    run_eq += total & 0xffffu;
  }
}

}  // namespace select
}  // namespace tri
