// Keep-highest selection for short rows: one warp per row.
//
// Same result as select_kernel (the top min(B, n) keys under the order score
// descending, index ascending; NaN lowest, -0 equal to +0; ascending indices
// out) -- page "The future-offset average in TriAttention can be
// precomputed", opening section: the cache keeps its highest-scoring keys
// within its budget.
//
// A serving cache that is re-compressed once per window of generated tokens
// (same page, "What it saves, and what it does not") holds rows only a little
// longer than the budget (B + the window, e.g. 2048 + 128), and there are
// thousands of them (layers x KV heads x sequences).  A CTA per row spends
// its time in a chain of block barriers; here a warp holds its row's
// order keys in registers (lane l owns keys 128 j + 4 l + q) and needs no
// barrier at all:
//  1. the finite range of the row (warp min/max) sets kWarpBins equal-width
//     value bins; a per-warp shared histogram and a suffix scan over the
//     lanes find the bin d that holds the B-th largest key;
//  2. the keys of bin d (a few dozen for smooth scores) are copied to shared
//     memory, and a bitwise search over them gives T, the B-th largest key,
//     exactly (the bins only narrow the search: binning is monotone in the
//     key, so every key of a higher bin is above T and every key of a lower
//     bin below it);
//  3. the emit walks the row in index order: per 128-key chunk, ballots give
//     each kept key its output slot and each key equal to T its tie rank, so
//     the `need` lowest-index ties are kept.
// Rows with no finite spread, or whose bin d overflows the candidate buffer
// (heavy duplication), run the bitwise search over the whole row instead.
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace tri {
namespace select {

constexpr int kWarpThreads = 256;                  // 8 rows per CTA
constexpr int kWarpRowsPerCta = kWarpThreads / 32;
constexpr int kWarpBins = 256;
constexpr int kWarpCand = 256;
constexpr int kWarpMaxRow = 4096;                  // 32 chunks of 128 keys, 128 keys per lane

struct __align__(16) WarpScratch {
  uint32_t hist[kWarpBins];
  uint32_t cand[kWarpCand];
};

__device__ __forceinline__ int value_bin_w(uint32_t key, float scale, float lo_s) {
  const int t = __float2int_rz(fmaf(key_value(key), scale, -lo_s));
  return min(max(t, 0), kWarpBins - 1);
}

// The largest t with #{x : x >= t} >= need, over the values each lane passes
// through `each` (need >= 1 and at most that many values).  Bits above
// those that all values in [lo, hi] share are fixed at once.
template <typename Each>
__device__ __forceinline__ uint32_t warp_kth_largest(Each each, uint32_t lo, uint32_t hi, uint32_t need) {
  const int fixed = lo == hi ? 32 : __clz(lo ^ hi);
  uint32_t prefix = fixed == 32 ? hi : (fixed ? (hi & (0xffffffffu << (32 - fixed))) : 0u);
  for (int bit = 31 - fixed; bit >= 0; --bit) {
    const uint32_t t = prefix | (1u << bit);
    uint32_t c = 0;
    each([&](uint32_t x) { c += x >= t; });
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= need) prefix = t;
  }
  return prefix;
}

// Select one row of n (B < n <= 128 J) scores; kept gets the B indices.
template <int J>
__device__ __forceinline__ void warp_select_row(const float* __restrict__ row, int n, int B, WarpScratch& S,
                                                int32_t* __restrict__ kept) {
  const int lane = threadIdx.x & 31;
  const int chunks = (n + 127) >> 7;               // warp-uniform
  uint32_t k[J][4];
  uint32_t fmin = 0xffffffffu, fmax = 0u;          // finite keys only
#pragma unroll
  for (int j = 0; j < J; ++j) {
    if (j < chunks) {
      const int i0 = 128 * j + 4 * lane;
      float v[4];
      if (i0 + 3 < n) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(row + i0));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = i0 + q < n ? __ldcg(row + i0 + q) : __uint_as_float(0x7fc00000u);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        k[j][q] = order_key(v[q]);                 // past the row: NaN's key 0, and never compared as a tie
        if (k[j][q] > kKeyNegInf && k[j][q] < kKeyPosInf) {
          fmin = min(fmin, k[j][q]);
          fmax = max(fmax, k[j][q]);
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) k[j][q] = 0u;
    }
  }
  fmin = __reduce_min_sync(0xffffffffu, fmin);
  fmax = __reduce_max_sync(0xffffffffu, fmax);

  auto each_key = [&](auto fn) {
#pragma unroll
    for (int j = 0; j < J; ++j)
      if (j < chunks) {
#pragma unroll
        for (int q = 0; q < 4; ++q) fn(k[j][q]);
      }
  };

  uint32_t need = static_cast<uint32_t>(B);
  uint32_t T = 0u;
  bool done = false;
  float scale = 0.f, lo_s = 0.f;
  bool binned = false;
  if (fmin < fmax) {
    const float lo = key_value(fmin);
    const float width = key_value(fmax) - lo;
    scale = static_cast<float>(kWarpBins) / width;
    lo_s = lo * scale;
    binned = width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s);
  }
  if (binned) {
#pragma unroll
    for (int b = lane; b < kWarpBins; b += 32) S.hist[b] = 0u;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < J; ++j)
      if (j < chunks) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (128 * j + 4 * lane + q < n) atomicAdd(&S.hist[value_bin_w(k[j][q], scale, lo_s)], 1u);
      }
    __syncwarp();
    // lane l owns bins [8 l, 8 l + 8); counts above a lane's bins by a suffix scan
    constexpr int kPer = kWarpBins / 32;
    static_assert(kPer == 8, "two 16-byte reads per lane");
    uint32_t h[kPer], mine = 0;
    const uint4 h0 = reinterpret_cast<const uint4*>(S.hist)[2 * lane];
    const uint4 h1 = reinterpret_cast<const uint4*>(S.hist)[2 * lane + 1];
    h[0] = h0.x; h[1] = h0.y; h[2] = h0.z; h[3] = h0.w;
    h[4] = h1.x; h[5] = h1.y; h[6] = h1.z; h[7] = h1.w;
#pragma unroll
    for (int e = 0; e < kPer; ++e) mine += h[e];
    uint32_t incl = mine;                          // sum over lanes >= this one
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const uint32_t above_lane = incl - mine;
    if (lane == 0) TRI_CHECK(incl == static_cast<uint32_t>(n));       // the bins total the row
    int d = -1;
    uint32_t above = 0;
    if (above_lane < need && incl >= need) {
      uint32_t acc = above_lane;
#pragma unroll
      for (int e = kPer - 1; e >= 0; --e) {
        if (d < 0 && acc + h[e] >= need) {
          d = kPer * lane + e;
          above = acc;
        }
        if (d < 0) acc += h[e];
      }
    }
    const uint32_t owner = __ballot_sync(0xffffffffu, d >= 0);
    const int src = __ffs(owner) - 1;              // exactly one lane: the bin totals reach n > B
    d = __shfl_sync(0xffffffffu, d, src);
    above = __shfl_sync(0xffffffffu, above, src);
    const uint32_t in_bin = S.hist[d];
    if (in_bin <= static_cast<uint32_t>(kWarpCand)) {
      // the bin's keys to shared memory, in any order (only their values matter)
      uint32_t base = 0, cmin = 0xffffffffu, cmax = 0u;
      const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
      for (int j = 0; j < J; ++j)
        if (j < chunks) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const bool in = 128 * j + 4 * lane + q < n && value_bin_w(k[j][q], scale, lo_s) == d;
            const uint32_t m = __ballot_sync(0xffffffffu, in);
            if (in) {
              S.cand[base + __popc(m & lt)] = k[j][q];
              cmin = min(cmin, k[j][q]);
              cmax = max(cmax, k[j][q]);
            }
            base += __popc(m);
          }
        }
      __syncwarp();
      cmin = __reduce_min_sync(0xffffffffu, cmin);
      cmax = __reduce_max_sync(0xffffffffu, cmax);
      need -= above;                               // 1 <= need <= in_bin
      const int nc = static_cast<int>(base);
      T = warp_kth_largest(
          [&](auto fn) {
#pragma unroll
            for (int m = 0; m < kWarpCand / 32; ++m)
              if (32 * m < nc && 32 * m + lane < nc) fn(S.cand[32 * m + lane]);
          },
          cmin, cmax, need);
      uint32_t gt = 0;
      for (int m = lane; m < nc; m += 32) gt += S.cand[m] > T;
      need -= __reduce_add_sync(0xffffffffu, gt);
      done = true;
    }
  }
  if (!done) {
    // whole-row search: every key counts (NaN keys and positions past the
    // row are 0, below every t >= 1 the search tests)
    T = warp_kth_largest(each_key, 0u, 0xffffffffu, need);
    uint32_t gt = 0;
    each_key([&](uint32_t x) { gt += x > T; });
    need -= __reduce_add_sync(0xffffffffu, gt);
  }
  // T is the B-th largest key; keep every key above it and the `need`
  // lowest-index keys equal to it.  Emit in index order.
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t slot = 0, ties = 0;
#pragma unroll
  for (int j = 0; j < J; ++j)
    if (j < chunks) {
      bool keep[4];
      bool tie[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = 128 * j + 4 * lane + q < n;
        keep[q] = valid && k[j][q] > T;
        tie[q] = valid && k[j][q] == T;
      }
      const bool any_tie = __any_sync(0xffffffffu, tie[0] || tie[1] || tie[2] || tie[3]);
      if (any_tie) {                               // warp-uniform
        uint32_t tm[4], before = 0, total = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tm[q] = __ballot_sync(0xffffffffu, tie[q]);
          before += __popc(tm[q] & lt);
          total += __popc(tm[q]);
        }
        uint32_t r = ties + before;                // tie rank of this lane's first tie
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (tie[q]) {
            keep[q] = r < need;
            ++r;
          }
        ties += total;
      }
      uint32_t km[4], before = 0, total = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        km[q] = __ballot_sync(0xffffffffu, keep[q]);
        before += __popc(km[q] & lt);
        total += __popc(km[q]);
      }
      uint32_t s = slot + before;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (keep[q]) kept[s++] = 128 * j + 4 * lane + q;
      slot += total;
    }
  if (lane == 0) TRI_CHECK(slot == static_cast<uint32_t>(B));         // exactly B kept
}

// One warp per unit, units [blockIdx.x * 8, ...): rows of at most 128 J keys.
template <int J>
__global__ void __launch_bounds__(kWarpThreads) select_warp_kernel(const __grid_constant__ Geom g, const Args a,
                                                                   int units) {
  __shared__ WarpScratch scratch[kWarpRowsPerCta];
  const int w = threadIdx.x >> 5;
  const int u = blockIdx.x * kWarpRowsPerCta + w;
  if (u >= units) return;                          // whole warps
  const int b = u % g.batch;
  const int n = g.len[b];
  const int B = a.B;
  int32_t* __restrict__ kept = a.kept + static_cast<int64_t>(u) * B;
  const int lane = threadIdx.x & 31;
  if (lane == 0) a.kept_count[u] = min(n, B);
  if (n <= B) {
    for (int i = lane; i < n; i += 32) kept[i] = i;
    return;
  }
  warp_select_row<J>(a.scores + static_cast<int64_t>(u) * g.score_stride, n, B, scratch[w], kept);
}

}  // namespace select
}  // namespace tri
