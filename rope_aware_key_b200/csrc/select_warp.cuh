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
// its time in a chain of block barriers; a warp per row needs none, and a
// few kilobytes of shared memory per warp let 32 or more rows run on an SM.
// Lane l owns keys 128 j + 4 l + q (one 16-byte load per 128-key chunk).
//  1. 256 evenly spaced scores of the row are binned into kWarpBins
//     equal-width value bins over their finite range (scores outside it
//     clamp to the end bins); a suffix scan of the bins over the lanes finds
//     the bins that hold the sample's ranks B/n * 256 -/+ (3 sigma + 4) from
//     the top: b_hi and b_lo.
//  2. One pass over the row counts the scores in bins above b_hi (all kept)
//     and gathers the scores in bins b_lo..b_hi, as order-preserving integer
//     keys, into a candidate buffer.  Binning is monotone in the score (NaN
//     in the lowest bin), so if the B-th largest lies among the candidates --
//     checked: above < B <= above + candidates -- a bitwise search over them
//     gives it exactly: T, and `need`, how many keys equal to T are kept.
//  3. The emit walks the row in index order: per chunk, ballots give each
//     kept key its output slot and each key equal to T its tie rank, so the
//     `need` lowest-index ties are kept.  These comparisons are made on the
//     floats themselves (-0 == +0; NaN, the lowest, compared apart).
// If the check fails (a pathological order, heavy duplication, no finite
// spread among the samples), a bitwise search over the whole row finds T.
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace tri {
namespace select {

constexpr int kWarpRows = 8;                       // rows (warps) per CTA
constexpr int kWarpThreads = kWarpRows * 32;
constexpr int kWarpBins = 256;
constexpr int kWarpSamples = 256;                  // 8 per lane
constexpr int kWarpCand = 768;
constexpr int kWarpMaxRow = 4096;

struct __align__(16) WarpScratch {
  uint32_t hist[kWarpBins];
  uint32_t cand[kWarpCand];                        // candidate keys (later: the evicted indices)
  int32_t cidx[kWarpCand];                         // their indices (rows that evict few keys)
};

// Value bin of a score: clamp(trunc(v * scale - lo_s), 0, kWarpBins - 1).
// The multiply-add and the saturating conversion are monotone; NaN converts
// to 0, scores below or above the binned range saturate to the end bins.
__device__ __forceinline__ int bin_of(float v, float scale, float lo_s) {
  const int t = __float2int_rz(fmaf(v, scale, -lo_s));
  return min(max(t, 0), kWarpBins - 1);
}

// Chunk j of a row (4 scores per lane); positions past the row read as 0.
__device__ __forceinline__ float4 row_chunk(const float* __restrict__ row, int n, int full, int j, int lane) {
  const int i0 = 128 * j + 4 * lane;
  if (j < full) return __ldg(reinterpret_cast<const float4*>(row + i0));
  float4 x;
  x.x = i0 < n ? __ldg(row + i0) : 0.f;
  x.y = i0 + 1 < n ? __ldg(row + i0 + 1) : 0.f;
  x.z = i0 + 2 < n ? __ldg(row + i0 + 2) : 0.f;
  x.w = i0 + 3 < n ? __ldg(row + i0 + 3) : 0.f;
  return x;
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

// Select one row of n > B scores (n <= kWarpMaxRow); kept gets the B indices.
__device__ __forceinline__ void warp_select_row(const float* __restrict__ row, int n, int B, WarpScratch& S,
                                                int32_t* __restrict__ kept) {
  const int lane = threadIdx.x & 31;
  const int chunks = (n + 127) >> 7;               // warp-uniform
  const int full = n >> 7;                          // chunks with no position past the row
  const uint32_t lt = (1u << lane) - 1u;
  auto valid = [&](int j, int q) { return j < full || 128 * j + 4 * lane + q < n; };

  // 1. samples: positions (p n) / 256, p = lane + 32 e
  float sv[kWarpSamples / 32];
  float mn = INFINITY, mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < kWarpSamples / 32; ++e) {
    sv[e] = __ldg(row + (((lane + 32 * e) * n) >> 8));
    const float f = fabsf(sv[e]) <= 3.402823466e38f ? sv[e] : NAN;    // finite only
    mn = fminf(mn, f);
    mx = fmaxf(mx, f);
  }
  const uint32_t kmin = __reduce_min_sync(0xffffffffu, order_key(mn));
  const uint32_t kmax = __reduce_max_sync(0xffffffffu, order_key(mx));
  float scale = 0.f, lo_s = 0.f;
  bool ok = false;
  if (kmin < kmax) {
    const float lo = key_value(kmin);
    const float width = key_value(kmax) - lo;
    scale = static_cast<float>(kWarpBins) / width;
    lo_s = lo * scale;
    ok = width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s);
  }
  uint32_t need = static_cast<uint32_t>(B);
  uint32_t T = 0u;
  if (ok) {
    for (int b = lane; b < kWarpBins; b += 32) S.hist[b] = 0u;
    __syncwarp();
#pragma unroll
    for (int e = 0; e < kWarpSamples / 32; ++e) atomicAdd(&S.hist[bin_of(sv[e], scale, lo_s)], 1u);
    __syncwarp();
    // lane l owns bins [8 l, 8 l + 8); sample counts above them by a suffix scan
    constexpr int kPer = kWarpBins / 32;
    static_assert(kPer == 8, "two 16-byte reads per lane");
    uint32_t h[kPer], mine = 0;
    const uint4 h0 = reinterpret_cast<const uint4*>(S.hist)[2 * lane];
    const uint4 h1 = reinterpret_cast<const uint4*>(S.hist)[2 * lane + 1];
    h[0] = h0.x; h[1] = h0.y; h[2] = h0.z; h[3] = h0.w;
    h[4] = h1.x; h[5] = h1.y; h[6] = h1.z; h[7] = h1.w;
#pragma unroll
    for (int e = 0; e < kPer; ++e) mine += h[e];
    uint32_t incl = mine;                          // samples in bins of lanes >= this one
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const uint32_t above_lane = incl - mine;
    // the bin of the R-th largest sample (R from 1); R < 1: the top bin, R > 256: bin 0
    auto bin_of_rank = [&](int R) {
      if (R < 1) return kWarpBins - 1;
      if (R > kWarpSamples) return 0;
      int d = -1;
      if (above_lane < static_cast<uint32_t>(R) && incl >= static_cast<uint32_t>(R)) {
        uint32_t acc = above_lane;
#pragma unroll
        for (int e = kPer - 1; e >= 0; --e) {
          if (d < 0 && acc + h[e] >= static_cast<uint32_t>(R)) d = kPer * lane + e;
          if (d < 0) acc += h[e];
        }
      }
      const uint32_t owner = __ballot_sync(0xffffffffu, d >= 0);
      return __shfl_sync(0xffffffffu, d, __ffs(owner) - 1);
    };
    const float r = static_cast<float>(B) * kWarpSamples / static_cast<float>(n);
    const float delta = 3.f * sqrtf(r * (1.f - r / kWarpSamples)) + 4.f;
    const int b_hi = bin_of_rank(static_cast<int>(floorf(r - delta)));
    const int b_lo = bin_of_rank(static_cast<int>(ceilf(r + delta)));

    if (b_lo == 0) {
      // Rows that evict few keys (B close to n): every key at or below bin
      // b_hi -- NaN included -- is a candidate, kept with its index, so the
      // evicted keys are all among the candidates.  One pass over the row;
      // the output is then written from the sorted list of evicted indices.
      const float U = b_hi >= kWarpBins - 1 ? INFINITY : (static_cast<float>(b_hi + 1) + lo_s) / scale;
      uint32_t above = 0, base = 0, cmin = 0xffffffffu, cmax = 0u;
      for (int j = 0; j < chunks; ++j) {
        const float4 x = row_chunk(row, n, full, j, lane);
        const float v[4] = {x.x, x.y, x.z, x.w};
        bool in[4];
        uint32_t before = 0, total = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool vq = valid(j, q);
          const bool up = v[q] > U;                // NaN: not above, a candidate
          above += vq && up;
          in[q] = vq && !up;
          const uint32_t m = __ballot_sync(0xffffffffu, in[q]);
          before += __popc(m & lt);
          total += __popc(m);
        }
        // index order: lanes, then q within a lane
        uint32_t pos = base + before;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (in[q]) {
            if (pos < static_cast<uint32_t>(kWarpCand)) {
              const uint32_t key = order_key(v[q]);
              S.cand[pos] = key;
              S.cidx[pos] = 128 * j + 4 * lane + q;
              cmin = min(cmin, key);
              cmax = max(cmax, key);
            }
            ++pos;
          }
        base += total;
      }
      above = __reduce_add_sync(0xffffffffu, above);
      if (above < static_cast<uint32_t>(B) && base <= static_cast<uint32_t>(kWarpCand) &&
          static_cast<uint32_t>(B) <= above + base) {
        __syncwarp();
        cmin = __reduce_min_sync(0xffffffffu, cmin);
        cmax = __reduce_max_sync(0xffffffffu, cmax);
        const int nc = static_cast<int>(base);
        const uint32_t need_c = static_cast<uint32_t>(B) - above;   // 1 <= need_c <= nc
        const uint32_t Tc = warp_kth_largest(
            [&](auto fn) {
              for (int m = lane; m < nc; m += 32) fn(S.cand[m]);
            },
            cmin, cmax, need_c);
        uint32_t gt = 0;
        for (int m = lane; m < nc; m += 32) gt += S.cand[m] > Tc;
        const uint32_t need_t = need_c - __reduce_add_sync(0xffffffffu, gt);   // ties to keep
        // the evicted indices, ascending: candidates below T, and ties past the
        // first need_t (written over the candidate keys already read)
        uint32_t ev = 0, ties = 0;
        for (int m0 = 0; m0 < nc; m0 += 32) {
          const int m = m0 + lane;
          const uint32_t k = m < nc ? S.cand[m] : 0xffffffffu;
          const int32_t i = m < nc ? S.cidx[m] : 0;
          const bool tie = m < nc && k == Tc;
          const uint32_t tm = __ballot_sync(0xffffffffu, tie);
          const bool out = m < nc && (k < Tc || (tie && ties + __popc(tm & lt) >= need_t));
          const uint32_t om = __ballot_sync(0xffffffffu, out);
          __syncwarp();                            // every lane has read its entry
          if (out) S.cand[ev + __popc(om & lt)] = static_cast<uint32_t>(i);
          ev += __popc(om);
          ties += __popc(tm);
        }
        __syncwarp();
        const int E = static_cast<int>(ev);
        if (lane == 0) TRI_CHECK(E == n - B);                     // exactly B kept
        const int32_t* evi = reinterpret_cast<const int32_t*>(S.cand);
        // kept[j] = j + #{t : ev[t] - t <= j} (ev[t] - t: the kept keys below
        // ev[t], non-decreasing); each lane writes a contiguous run of slots
        const int per = (((B + 31) >> 5) + 3) & ~3;
        const int jb = min(B, lane * per), je = min(B, jb + per);
        int a = 0, c = E;                          // first t with ev[t] - t > jb
        while (a < c) {
          const int mid = (a + c) >> 1;
          if (evi[mid] - mid <= jb) a = mid + 1;
          else c = mid;
        }
        int e = a;
        const bool vec = ((reinterpret_cast<uintptr_t>(kept + jb) & 15u) == 0) && ((je - jb) & 3) == 0;
        if (vec) {
          for (int j = jb; j < je; j += 4) {
            int o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              while (e < E && evi[e] - e <= j + q) ++e;
              o[q] = j + q + e;
            }
            *reinterpret_cast<int4*>(kept + j) = make_int4(o[0], o[1], o[2], o[3]);
          }
        } else {
          for (int j = jb; j < je; ++j) {
            while (e < E && evi[e] - e <= j) ++e;
            kept[j] = j + e;
          }
        }
        return;
      }
      ok = false;                                  // the whole-row search below
    } else {
      // 2. one pass: count the scores above b_hi, gather those in [b_lo, b_hi]
      uint32_t above = 0, base = 0, cmin = 0xffffffffu, cmax = 0u;
      for (int j = 0; j < chunks; ++j) {
        const float4 x = row_chunk(row, n, full, j, lane);
        const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int bq = bin_of(v[q], scale, lo_s);
          const bool vq = valid(j, q);
          above += vq && bq > b_hi;
          const bool in = vq && bq >= b_lo && bq <= b_hi;
          const uint32_t m = __ballot_sync(0xffffffffu, in);
          const uint32_t pos = base + __popc(m & lt);
          if (in && pos < static_cast<uint32_t>(kWarpCand)) {
            const uint32_t key = order_key(v[q]);
            S.cand[pos] = key;
            cmin = min(cmin, key);
            cmax = max(cmax, key);
          }
          base += __popc(m);
        }
      }
      above = __reduce_add_sync(0xffffffffu, above);
      ok = above < static_cast<uint32_t>(B) && static_cast<uint32_t>(B) <= above + base &&
           base <= static_cast<uint32_t>(kWarpCand);
      if (ok) {
        __syncwarp();
        cmin = __reduce_min_sync(0xffffffffu, cmin);
        cmax = __reduce_max_sync(0xffffffffu, cmax);
        need -= above;                               // 1 <= need <= candidates
        const int nc = static_cast<int>(base);
        T = warp_kth_largest(
            [&](auto fn) {
              for (int m = lane; m < nc; m += 32) fn(S.cand[m]);
            },
            cmin, cmax, need);
        uint32_t gt = 0;
        for (int m = lane; m < nc; m += 32) gt += S.cand[m] > T;
        need -= __reduce_add_sync(0xffffffffu, gt);
      }
    }
  }
  if (!ok) {
    // whole-row search: every key of the row counts (NaN keys are 0, below
    // every t >= 1 the search tests)
    auto each_key = [&](auto fn) {
      for (int j = 0; j < chunks; ++j) {
        const float4 x = row_chunk(row, n, full, j, lane);
        const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (valid(j, q)) fn(order_key(v[q]));
      }
    };
    need = static_cast<uint32_t>(B);
    T = warp_kth_largest(each_key, 0u, 0xffffffffu, need);
    uint32_t gt = 0;
    each_key([&](uint32_t x) { gt += x > T; });
    need -= __reduce_add_sync(0xffffffffu, gt);
  }

  // 3. T is the B-th largest key; keep every key above it and the `need`
  // lowest-index keys equal to it.  Emit in index order, comparing floats:
  // above T means a greater float (every number, if T is NaN's key), equal
  // to T a float that compares equal (NaN, if T is NaN's key).
  const bool t_nan = T == 0u;
  const float tf = key_value(T);
  uint32_t slot = 0, ties = 0;
  for (int j = 0; j < chunks; ++j) {
    const float4 x = row_chunk(row, n, full, j, lane);
    const float v[4] = {x.x, x.y, x.z, x.w};
    bool keep[4], tie[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool vq = valid(j, q);
      const bool nan = v[q] != v[q];
      keep[q] = vq && (t_nan ? !nan : v[q] > tf);
      tie[q] = vq && (t_nan ? nan : v[q] == tf);
    }
    if (__any_sync(0xffffffffu, tie[0] || tie[1] || tie[2] || tie[3])) {   // warp-uniform
      uint32_t before = 0, total = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t tm = __ballot_sync(0xffffffffu, tie[q]);
        before += __popc(tm & lt);
        total += __popc(tm);
      }
      uint32_t rk = ties + before;                 // tie rank of this lane's first tie
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (tie[q]) {
          keep[q] = rk < need;
          ++rk;
        }
      ties += total;
    }
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t km = __ballot_sync(0xffffffffu, keep[q]);
      before += __popc(km & lt);
      total += __popc(km);
    }
    uint32_t s = slot + before;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (keep[q]) kept[s++] = 128 * j + 4 * lane + q;
    slot += total;
  }
  if (lane == 0) TRI_CHECK(slot == static_cast<uint32_t>(B));         // exactly B kept
}

constexpr size_t kWarpSmemBytes = kWarpRows * sizeof(WarpScratch);

// One warp per unit, units [blockIdx.x * kWarpRows, ...): rows of at most
// kWarpMaxRow keys.  Dynamic shared memory: kWarpSmemBytes.
__global__ void __launch_bounds__(kWarpThreads) select_warp_kernel(const __grid_constant__ Geom g, const Args a,
                                                                   int units) {
  extern __shared__ float4 select_warp_dyn[];
  WarpScratch* scratch = reinterpret_cast<WarpScratch*>(select_warp_dyn);
  const int w = threadIdx.x >> 5;
  const int u = blockIdx.x * kWarpRows + w;
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
  warp_select_row(a.scores + static_cast<int64_t>(u) * g.score_stride, n, B, scratch[w], kept);
}

}  // namespace select
}  // namespace tri
