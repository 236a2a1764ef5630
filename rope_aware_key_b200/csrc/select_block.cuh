// Keep-highest selection for long rows: one CTA of 16 warps per row, with a
// fixed, small amount of shared memory whatever the row length.
//
// Same result as the other selection kernels (the top min(B, n) keys under
// the order score descending, index ascending; NaN lowest, -0 equal to +0;
// ascending indices out) -- page "The future-offset average in TriAttention
// can be precomputed", opening section: the cache keeps its highest-scoring
// keys within its budget.
//
// Warp w owns a contiguous segment of the row (whole 128-key chunks; lane l
// reads keys 128 j + 4 l + q of its chunks).  The row is read twice:
//  1. 4096 evenly spaced scores, binned into kBlkBins equal-width bins over
//     their finite range (scores outside it clamp to the end bins), give the
//     bins b_hi / b_lo that hold the sample's ranks B/n * 4096 -/+
//     (3 sigma + 4) from the top;
//  2. pass one: each warp counts its scores in bins above b_hi (all kept) and
//     gathers those in bins b_lo..b_hi, as order-preserving integer keys,
//     into its own candidate buffer.  If the B-th largest lies among the
//     candidates (above < B <= above + candidates, and no buffer overflowed),
//     a second histogram over the candidates' own range narrows it to one
//     fine bin, whose few keys one warp searches bitwise: T, the B-th largest
//     key, and `need`, how many keys equal to T are kept;
//  3. each warp counts, from its candidates, its keys above T and equal to T;
//     prefix sums over the warps give every warp its first output slot and
//     its first tie rank;
//  4. pass two: each warp emits its segment in index order (ballots per
//     chunk), keeping every key above T and the `need` lowest-index ties.
// Binning is monotone in the score (NaN in the lowest bin), so every key of a
// higher bin is above every key of a lower one, and the result is exact.  If
// the check fails (a pathological order, heavy duplication, no finite spread
// among the samples), a bitwise search over the whole row (one pass per bit)
// finds T instead, and the counts of step 3 come from the row.
#pragma once

#include "common.cuh"
#include "select.cuh"
#include "select_warp.cuh"

namespace tri {
namespace select {

constexpr int kBlkWarps = 16;
constexpr int kBlkThreads = kBlkWarps * 32;
constexpr int kBlkSamples = 4096;                  // 8 per thread
constexpr int kBlkBins = 2048;                     // 4 per thread
constexpr int kBlkCand = 512;                      // candidates per warp
constexpr int kBlkFew = 256;                       // keys of the fine bin searched by one warp

struct BlkScratch {
  uint32_t hist[kBlkBins];                         // sample bins, then the candidates' fine bins
  uint32_t cand[kBlkWarps][kBlkCand];
  uint32_t few[kBlkFew];
  uint32_t w_above[kBlkWarps], w_cand[kBlkWarps], w_gt[kBlkWarps], w_eq[kBlkWarps];
  uint32_t w_min[kBlkWarps], w_max[kBlkWarps];
  uint32_t scan[kBlkWarps];
  int sel[4];                                      // broadcasts: bins found by the owning thread
  uint32_t t_key, t_need, n_few;
};

// Over the block: bins [kPer t, kPer t + kPer) belong to thread t.  Returns the
// bin holding the R-th largest count (R from 1); R < 1: the top bin,
// R > total: bin 0.  Contains barriers: call from every thread.
template <int kPer>
__device__ __forceinline__ int blk_bin_of_rank(const uint32_t* hist, int R, uint32_t total, BlkScratch& S, int slot) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  uint32_t h[kPer], mine = 0;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    h[e] = hist[kPer * t + e];
    mine += h[e];
  }
  uint32_t incl = mine;                            // over the threads >= t of this warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += y;
  }
  if (lane == 0) S.scan[warp] = incl;              // the warp's total
  __syncthreads();
  uint32_t higher = 0;                             // warps above this one
  for (int w = warp + 1; w < kBlkWarps; ++w) higher += S.scan[w];
  incl += higher;
  const uint32_t above_t = incl - mine;
  if (R < 1) {
    if (t == 0) S.sel[slot] = kPer * kBlkThreads - 1;
  } else if (static_cast<uint32_t>(R) > total) {
    if (t == 0) S.sel[slot] = 0;
  } else if (above_t < static_cast<uint32_t>(R) && incl >= static_cast<uint32_t>(R)) {
    uint32_t acc = above_t;
    int d = -1;
#pragma unroll
    for (int e = kPer - 1; e >= 0; --e) {
      if (d < 0 && acc + h[e] >= static_cast<uint32_t>(R)) {
        d = kPer * t + e;
        S.sel[slot + 1] = static_cast<int>(acc);   // count above the bin
      }
      if (d < 0) acc += h[e];
    }
    S.sel[slot] = d;
  }
  __syncthreads();
  const int d = S.sel[slot];
  __syncthreads();                                 // scan and sel may be rewritten next
  return d;
}

// Select one row of n > B scores; kept gets the B indices.
__device__ __forceinline__ void block_select_row(const float* __restrict__ row, int n, int B, BlkScratch& S,
                                                 int32_t* __restrict__ kept) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int chunks = (n + 127) >> 7;
  const int full = n >> 7;
  const int per_warp = (chunks + kBlkWarps - 1) / kBlkWarps;
  const int j0 = min(chunks, warp * per_warp), j1 = min(chunks, j0 + per_warp);
  auto valid = [&](int j, int q) { return j < full || 128 * j + 4 * lane + q < n; };

  // 1. samples and their finite range
  float sv[kBlkSamples / kBlkThreads];
  float mn = INFINITY, mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < kBlkSamples / kBlkThreads; ++e) {
    const int64_t p = t + static_cast<int64_t>(kBlkThreads) * e;
    sv[e] = __ldg(row + ((p * n) >> 12));
    const float f = fabsf(sv[e]) <= 3.402823466e38f ? sv[e] : NAN;    // finite only
    mn = fminf(mn, f);
    mx = fmaxf(mx, f);
  }
  uint32_t kmn = __reduce_min_sync(0xffffffffu, order_key(mn));
  uint32_t kmx = __reduce_max_sync(0xffffffffu, order_key(mx));
  if (lane == 0) {
    S.w_min[warp] = kmn;
    S.w_max[warp] = kmx;
  }
  for (int b = t; b < kBlkBins; b += kBlkThreads) S.hist[b] = 0u;
  __syncthreads();
  kmn = 0xffffffffu;
  kmx = 0u;
  for (int w = 0; w < kBlkWarps; ++w) {
    kmn = min(kmn, S.w_min[w]);
    kmx = max(kmx, S.w_max[w]);
  }
  float scale = 0.f, lo_s = 0.f;
  bool ok = false;
  if (kmn < kmx) {
    const float lo = key_value(kmn);
    const float width = key_value(kmx) - lo;
    scale = static_cast<float>(kBlkBins) / width;
    lo_s = lo * scale;
    ok = width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s);
  }
  auto bin = [&](float v) {
    const int x = __float2int_rz(fmaf(v, scale, -lo_s));
    return min(max(x, 0), kBlkBins - 1);
  };
  uint32_t T = 0u, need = static_cast<uint32_t>(B);
  uint32_t above_w = 0, gt_w = 0, eq_w = 0;        // this warp: keys above the bins, above T, equal to T
  if (ok) {                                        // block-uniform
#pragma unroll
    for (int e = 0; e < kBlkSamples / kBlkThreads; ++e) atomicAdd(&S.hist[bin(sv[e])], 1u);
    __syncthreads();
    const float r = static_cast<float>(B) * kBlkSamples / static_cast<float>(n);
    const float delta = 3.f * sqrtf(r * (1.f - r / kBlkSamples)) + 4.f;
    const int b_hi = blk_bin_of_rank<kBlkBins / kBlkThreads>(S.hist, static_cast<int>(floorf(r - delta)),
                                                             kBlkSamples, S, 0);
    const int b_lo = blk_bin_of_rank<kBlkBins / kBlkThreads>(S.hist, static_cast<int>(ceilf(r + delta)),
                                                             kBlkSamples, S, 2);
    // 2. pass one over this warp's segment
    uint32_t base = 0, cmin = 0xffffffffu, cmax = 0u;
    uint32_t* cand = S.cand[warp];
    for (int j = j0; j < j1; ++j) {
      const float4 x = row_chunk(row, n, full, j, lane);
      const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int bq = bin(v[q]);
        const bool vq = valid(j, q);
        above_w += vq && bq > b_hi;
        const bool in = vq && bq >= b_lo && bq <= b_hi;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        const uint32_t pos = base + __popc(m & lt);
        if (in && pos < static_cast<uint32_t>(kBlkCand)) {
          const uint32_t key = order_key(v[q]);
          cand[pos] = key;
          cmin = min(cmin, key);
          cmax = max(cmax, key);
        }
        base += __popc(m);
      }
    }
    above_w = __reduce_add_sync(0xffffffffu, above_w);
    cmin = __reduce_min_sync(0xffffffffu, cmin);
    cmax = __reduce_max_sync(0xffffffffu, cmax);
    if (lane == 0) {
      S.w_above[warp] = above_w;
      S.w_cand[warp] = base;
      S.w_min[warp] = cmin;
      S.w_max[warp] = cmax;
    }
    __syncthreads();
    uint32_t above = 0, ncand = 0;
    bool fits = true;
    cmin = 0xffffffffu;
    cmax = 0u;
    for (int w = 0; w < kBlkWarps; ++w) {
      above += S.w_above[w];
      ncand += S.w_cand[w];
      fits = fits && S.w_cand[w] <= static_cast<uint32_t>(kBlkCand);
      cmin = min(cmin, S.w_min[w]);
      cmax = max(cmax, S.w_max[w]);
    }
    ok = fits && above < static_cast<uint32_t>(B) && static_cast<uint32_t>(B) <= above + ncand;
    if (ok) {
      need -= above;                               // 1 <= need <= ncand
      const int nc_w = static_cast<int>(S.w_cand[warp]);
      // fine bins over the candidates' own value range (block-uniform choice)
      float fscale = 0.f, flo_s = 0.f;
      bool fine = false;
      if (cmin < cmax && cmin > kKeyNegInf && cmax < kKeyPosInf) {
        const float lo = key_value(cmin);
        const float width = key_value(cmax) - lo;
        fscale = static_cast<float>(kBlkBins) / width;
        flo_s = lo * fscale;
        fine = width > 0.f && isfinite(width) && isfinite(fscale) && fscale > 0.f && isfinite(flo_s);
      }
      uint32_t lo_key = cmin, hi_key = cmax;
      int d2 = -1;
      if (fine) {
        auto fbin = [&](uint32_t k) {
          const int x = __float2int_rz(fmaf(key_value(k), fscale, -flo_s));
          return min(max(x, 0), kBlkBins - 1);
        };
        for (int b = t; b < kBlkBins; b += kBlkThreads) S.hist[b] = 0u;
        __syncthreads();
        for (int m = lane; m < nc_w; m += 32) atomicAdd(&S.hist[fbin(S.cand[warp][m])], 1u);
        __syncthreads();
        d2 = blk_bin_of_rank<kBlkBins / kBlkThreads>(S.hist, static_cast<int>(need), ncand, S, 0);
        const uint32_t above2 = static_cast<uint32_t>(S.sel[1]);
        const uint32_t in2 = S.hist[d2];
        // one warp searches the fine bin's keys (if they fit), else every candidate
        if (warp == 0) {
          uint32_t nf = 0;
          if (in2 <= static_cast<uint32_t>(kBlkFew)) {
            for (int w = 0; w < kBlkWarps; ++w) {
              const int nw = static_cast<int>(S.w_cand[w]);
              for (int m0 = 0; m0 < nw; m0 += 32) {
                const int m = m0 + lane;
                const uint32_t k = m < nw ? S.cand[w][m] : 0u;
                const bool in = m < nw && fbin(k) == d2;
                const uint32_t bm = __ballot_sync(0xffffffffu, in);
                if (in) S.few[nf + __popc(bm & lt)] = k;
                nf += __popc(bm);
              }
            }
            __syncwarp();
            uint32_t fmin = 0xffffffffu, fmax = 0u;
            for (int m = lane; m < static_cast<int>(nf); m += 32) {
              fmin = min(fmin, S.few[m]);
              fmax = max(fmax, S.few[m]);
            }
            fmin = __reduce_min_sync(0xffffffffu, fmin);
            fmax = __reduce_max_sync(0xffffffffu, fmax);
            const uint32_t need2 = need - above2;
            const int nfi = static_cast<int>(nf);
            const uint32_t Tw = warp_kth_largest(
                [&](auto fn) {
                  for (int m = lane; m < nfi; m += 32) fn(S.few[m]);
                },
                fmin, fmax, need2);
            if (lane == 0) {
              S.t_key = Tw;
              S.n_few = 1u;
            }
          } else if (lane == 0) {
            S.n_few = 0u;                           // too crowded: search every candidate below
          }
        }
        __syncthreads();
        lo_key = cmin;
        hi_key = cmax;
        if (S.n_few) d2 = -2;                       // found
      }
      if (d2 != -2) {
        // every candidate, one warp (few distinct values, or a crowded fine bin)
        if (warp == 0) {
          const uint32_t Tw = warp_kth_largest(
              [&](auto fn) {
                for (int w = 0; w < kBlkWarps; ++w) {
                  const int nw = static_cast<int>(S.w_cand[w]);
                  for (int m = lane; m < nw; m += 32) fn(S.cand[w][m]);
                }
              },
              lo_key, hi_key, need);
          if (lane == 0) S.t_key = Tw;
        }
        __syncthreads();
      }
      T = S.t_key;
      // 3. this warp's candidates above T and equal to T
      for (int m = lane; m < nc_w; m += 32) {
        gt_w += S.cand[warp][m] > T;
        eq_w += S.cand[warp][m] == T;
      }
      gt_w = above_w + __reduce_add_sync(0xffffffffu, gt_w);
      eq_w = __reduce_add_sync(0xffffffffu, eq_w);
    }
  }
  if (!ok) {                                       // block-uniform
    // bitwise search over the whole row: one pass and one block sum per bit
    auto count_ge = [&](uint32_t th) {
      uint32_t c = 0;
      for (int j = j0; j < j1; ++j) {
        const float4 x = row_chunk(row, n, full, j, lane);
        const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) c += valid(j, q) && order_key(v[q]) >= th;
      }
      return __reduce_add_sync(0xffffffffu, c);
    };
    uint32_t prefix = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t th = prefix | (1u << bit);
      const uint32_t c = count_ge(th);
      __syncthreads();                             // the previous bit's totals have been read
      if (lane == 0) S.w_above[warp] = c;
      __syncthreads();
      uint32_t tot = 0;
      for (int w = 0; w < kBlkWarps; ++w) tot += S.w_above[w];
      if (tot >= static_cast<uint32_t>(B)) prefix = th;
    }
    T = prefix;
    gt_w = 0;
    eq_w = 0;
    for (int j = j0; j < j1; ++j) {
      const float4 x = row_chunk(row, n, full, j, lane);
      const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t k = order_key(v[q]);
        gt_w += valid(j, q) && k > T;
        eq_w += valid(j, q) && k == T;
      }
    }
    gt_w = __reduce_add_sync(0xffffffffu, gt_w);
    eq_w = __reduce_add_sync(0xffffffffu, eq_w);
  }
  // 3'. every warp's keys above T and equal to T: the ties to keep, and this
  // warp's first output slot and first tie rank
  __syncthreads();
  if (lane == 0) {
    S.w_gt[warp] = gt_w;
    S.w_eq[warp] = eq_w;
  }
  __syncthreads();
  uint32_t gt_all = 0;
  for (int w = 0; w < kBlkWarps; ++w) gt_all += S.w_gt[w];
  need = static_cast<uint32_t>(B) - gt_all;        // ties to keep, lowest indices first
  uint32_t slot = 0, ties = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t e_before = ties;
    ties += S.w_eq[w];
    const uint32_t e_keep = ties <= need ? S.w_eq[w] : (e_before < need ? need - e_before : 0u);
    slot += S.w_gt[w] + e_keep;
  }
  // 4. pass two: emit this warp's segment in index order
  const bool t_nan = T == 0u;
  const float tf = key_value(T);
  for (int j = j0; j < j1; ++j) {
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
      uint32_t rk = ties + before;
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
  if (warp == kBlkWarps - 1 && lane == 0) TRI_CHECK(slot == static_cast<uint32_t>(B));   // exactly B kept
}

// One CTA per unit.
__global__ void __launch_bounds__(kBlkThreads, 2) select_block_kernel(const __grid_constant__ Geom g, const Args a) {
  extern __shared__ float4 select_block_dyn[];
  BlkScratch& S = *reinterpret_cast<BlkScratch*>(select_block_dyn);
  const int u = blockIdx.x;
  const int b = u % g.batch;
  const int n = g.len[b];
  const int B = a.B;
  int32_t* __restrict__ kept = a.kept + static_cast<int64_t>(u) * B;
  if (threadIdx.x == 0) a.kept_count[u] = min(n, B);
  if (n <= B) {
    for (int i = threadIdx.x; i < n; i += kBlkThreads) kept[i] = i;
    return;
  }
  block_select_row(a.scores + static_cast<int64_t>(u) * g.score_stride, n, B, S, kept);
}

}  // namespace select
}  // namespace tri
