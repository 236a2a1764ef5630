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
// its time in a chain of block barriers; a warp per row needs none, and with
// 5 KB of shared memory per warp, CTAs of 4 rows fill an SM seven at a time.
// Every decision is made on order-preserving integer keys of the fp32 scores
// (NaN lowest), so the result is exact:
//  1. of 256 evenly spaced scores of the row (8 per lane), the ones at ranks
//     B/n * 256 -/+ (4 sigma + 8) from the top give two keys U >= L that
//     bracket the B-th largest key for any but a pathological order of the
//     scores; each is located to two 8-bit digits of the samples' key range
//     (a shared histogram per digit), U at the top of its bin and L at the
//     bottom, which only widens the bracket;
//  2. one pass over the row counts the keys above U (all kept) and gathers
//     the keys in [L, U] into a candidate buffer, in index order (the
//     comparisons are made on the floats; the candidates are stored as float
//     bits and turned into keys afterwards).  When L would fall below the
//     sample (rows that evict few keys), every key up to U is a candidate
//     and is gathered with its index;
//  3. if the B-th largest lies among the candidates (above < B <= above +
//     candidates), a radix search over them (8-bit digits, a shared histogram
//     per digit) gives it exactly: T, and `need`, how many keys equal to T
//     are kept (the lowest-index ones);
//  4. rows that evict few keys: the evicted positions (candidates below T,
//     and ties past the first `need`) are marked in a bitmap of the row, and
//     a scan of its words' counts gives, for every kept position p, its slot
//     p - #{evicted before p}; the kept indices are written position chunk by
//     position chunk, with no second pass over the scores.  Other rows: a
//     second pass emits the kept keys in index order (ballots per 128-key
//     chunk).
// If the check fails (a pathological order, heavy duplication), the radix
// search runs over the whole row instead (one pass per digit).  In-place
// compaction of rows that move few keys runs in the same kernel: the warp
// fills the row's holes right after selecting it (warp_fill_row).
#pragma once

#include <type_traits>

#include "common.cuh"
#include "compact.cuh"
#include "select.cuh"

namespace tri {
namespace select {

constexpr int kWarpRows = 4;                       // rows (warps) per CTA
constexpr int kWarpThreads = kWarpRows * 32;
constexpr int kWarpSamples = 256;                  // 8 per lane
constexpr int kWarpCand = 512;
constexpr int kWarpMaxRow = 4096;
constexpr int kWarpBatch = 4;                     // chunks whose loads are in flight together (6 or 8: the same time)
constexpr int kWarpCtasPerSm = 7;                 // register budget: 72 per thread

struct __align__(16) WarpScratch {
  uint32_t hist[256];                              // the radix digits; then the evicted bitmap and its word counts
  uint32_t cand[kWarpCand];                        // candidate keys (later: the fill's row offsets)
  int32_t cidx[kWarpCand];                         // their indices (rows that evict few keys; later: the holes)
};
constexpr size_t kWarpSmemBytes = kWarpRows * sizeof(WarpScratch);

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

// The need-th largest (need >= 1) of the keys in [lo, hi] among the keys the
// lanes pass through `each` (at least `need` of them lie in [lo, hi]), by
// 8-bit digits of key - lo, most significant first: each digit's histogram
// (hist, 256 words) picks the bin that holds the rank.  *need becomes the
// rank of the result among the keys equal to it.  With max_digits, the search
// stops after that many digits: the result is then in [returned, *hi_out].
template <typename Each>
__device__ __forceinline__ uint32_t warp_radix_kth(Each each, uint32_t lo, uint32_t hi, uint32_t* need,
                                                   uint32_t* hist, int max_digits = 4,
                                                   uint32_t* hi_out = nullptr) {
  const int lane = threadIdx.x & 31;
  for (int digit = 0; lo < hi && digit < max_digits; ++digit) {
    const int bits = 32 - __clz(hi - lo);
    const int shift = bits > 8 ? bits - 8 : 0;
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 8; ++e) hist[32 * e + lane] = 0u;
    __syncwarp();
    each([&](uint32_t k) {
      if (k >= lo && k <= hi) atomicAdd(&hist[(k - lo) >> shift], 1u);
    });
    __syncwarp();
    // lane l owns digits [8 l, 8 l + 8); counts above a lane's digits by a suffix scan
    const uint4 h0 = reinterpret_cast<const uint4*>(hist)[2 * lane];
    const uint4 h1 = reinterpret_cast<const uint4*>(hist)[2 * lane + 1];
    const uint32_t h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    uint32_t mine = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) mine += h[e];
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const uint32_t above_lane = incl - mine;
    int d = -1;
    uint32_t above = 0;
    if (above_lane < *need && incl >= *need) {
      uint32_t acc = above_lane;
#pragma unroll
      for (int e = 7; e >= 0; --e) {
        if (d < 0 && acc + h[e] >= *need) {
          d = 8 * lane + e;
          above = acc;
        }
        if (d < 0) acc += h[e];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, d >= 0)) - 1;
    d = __shfl_sync(0xffffffffu, d, src);
    *need -= __shfl_sync(0xffffffffu, above, src);
    lo += static_cast<uint32_t>(d) << shift;
    const uint64_t top = static_cast<uint64_t>(lo) + ((uint64_t{1} << shift) - 1u);   // no wrap near 2^32
    hi = top < hi ? static_cast<uint32_t>(top) : hi;
  }
  if (hi_out) *hi_out = hi;
  return lo;
}

// Select one row of n > B scores (n <= kWarpMaxRow); kept gets the B indices.
// Returns true when the evicted positions are left as a bitmap in S.hist
// (word w: positions 32 w .. 32 w + 31) with, in S.hist + 128, the count of
// evicted positions before each word.
__device__ __forceinline__ bool warp_select_row(const float* __restrict__ row, int n, int B, WarpScratch& S,
                                                int32_t* __restrict__ kept) {
  const int lane = threadIdx.x & 31;
  const int chunks = (n + 127) >> 7;               // warp-uniform
  const int full = n >> 7;                          // chunks with no position past the row
  const uint32_t lt = (1u << lane) - 1u;
  auto valid = [&](int j, int q) { return j < full || 128 * j + 4 * lane + q < n; };

  // 1. the bracket from the sample: two of its order statistics
  uint32_t x[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = order_key(__ldg(row + (((8 * lane + e) * n) >> 8)));
  uint32_t kmin = x[0], kmax = x[0];
#pragma unroll
  for (int e = 1; e < 8; ++e) {
    kmin = min(kmin, x[e]);
    kmax = max(kmax, x[e]);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const float r = static_cast<float>(B) * kWarpSamples / static_cast<float>(n);
  const float delta = 4.f * sqrtf(r * (1.f - r / kWarpSamples)) + 8.f;
  const int r_hi = static_cast<int>(floorf(r - delta)), r_lo = static_cast<int>(ceilf(r + delta));
  // the r_hi-th and r_lo-th largest samples (ranks counted from the top), to
  // two 8-bit digits of the samples' key range: U is taken at the top of its
  // last bin and L at the bottom, so each bound only widens the bracket (by
  // less than 2^-15 of the samples' key range)
  auto each_sample = [&](auto fn) {
#pragma unroll
    for (int e = 0; e < 8; ++e) fn(x[e]);
  };
  uint32_t U = 0xffffffffu, L0 = 0u;
  if (r_hi >= 1) {
    uint32_t rank = static_cast<uint32_t>(r_hi);
    warp_radix_kth(each_sample, kmin, kmax, &rank, S.hist, 2, &U);
  }
  if (r_lo <= kWarpSamples) {
    uint32_t rank = static_cast<uint32_t>(r_lo);
    L0 = warp_radix_kth(each_sample, kmin, kmax, &rank, S.hist, 2);
  }
  // rows that evict few keys (no lower bound; also when the bound is NaN's key)
  const bool few = L0 == 0u;
  // the same bounds as floats: above U is v > uf (NaN never is), in [L, U] is
  // !(v > uf) && v >= lf (every number when L is -inf's key)
  const float uf = U == 0xffffffffu ? INFINITY : key_value(U);
  const float lf = key_value(L0);

  // 2. one pass gathers the candidates, in index order: every key up to U
  // (rows that evict few keys: all the others are kept, so `above` is n minus
  // the candidates), else the keys in [L, U], counting those above U.  The
  // candidates are stored as float bits (with their indices when few) and
  // turned into keys afterwards; the loads of kWarpBatch chunks are issued
  // before any of them is used.
  uint32_t base = 0, upc = 0;
  auto collect = [&](auto few_c) {
    constexpr bool kFew = decltype(few_c)::value;
    for (int j0 = 0; j0 < chunks; j0 += kWarpBatch) {
      float4 xb[kWarpBatch];
#pragma unroll
      for (int i = 0; i < kWarpBatch; ++i)
        if (j0 + i < chunks) xb[i] = row_chunk(row, n, full, j0 + i, lane);
#pragma unroll
      for (int i = 0; i < kWarpBatch; ++i) {
        const int j = j0 + i;
        if (j >= chunks) break;                    // warp-uniform
        const float v[4] = {xb[i].x, xb[i].y, xb[i].z, xb[i].w};
        bool in[4];
        uint32_t cnt = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool vq = valid(j, q);
          const bool up = v[q] > uf;
          in[q] = vq && !up && (kFew || v[q] >= lf);
          if constexpr (!kFew) upc += __popc(__ballot_sync(0xffffffffu, vq && up));
          cnt += in[q];
        }
        // index order is lanes, then q: the lane's first slot is the
        // candidates of the lanes before it (cnt <= 4, summed by bit planes)
        const uint32_t b0 = __ballot_sync(0xffffffffu, cnt & 1u), b1 = __ballot_sync(0xffffffffu, cnt & 2u),
                       b2 = __ballot_sync(0xffffffffu, cnt & 4u);
        uint32_t pos = base + __popc(b0 & lt) + 2u * __popc(b1 & lt) + 4u * __popc(b2 & lt);
        base += __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (in[q]) {
            if (pos < static_cast<uint32_t>(kWarpCand)) {
              S.cand[pos] = __float_as_uint(v[q]);
              if (kFew) S.cidx[pos] = 128 * j + 4 * lane + q;
            }
            ++pos;
          }
      }
    }
  };
  if (few)
    collect(std::true_type());
  else
    collect(std::false_type());
  const uint32_t above = few ? static_cast<uint32_t>(n) - base : upc;
  const bool ok = above < static_cast<uint32_t>(B) && static_cast<uint32_t>(B) <= above + base &&
                  base <= static_cast<uint32_t>(kWarpCand);
  uint32_t T, need;
  if (ok) {
    __syncwarp();
    const int nc = static_cast<int>(base);
    uint32_t cmin = 0xffffffffu, cmax = 0u;
    for (int m = lane; m < nc; m += 32) {
      const uint32_t k = order_key(__uint_as_float(S.cand[m]));
      S.cand[m] = k;
      cmin = min(cmin, k);
      cmax = max(cmax, k);
    }
    cmin = __reduce_min_sync(0xffffffffu, cmin);
    cmax = __reduce_max_sync(0xffffffffu, cmax);
    __syncwarp();
    need = static_cast<uint32_t>(B) - above;       // 1 <= need <= base
    // 3. the exact threshold among the candidates; need becomes the ties to keep
    T = warp_radix_kth(
        [&](auto fn) {
          for (int m = lane; m < nc; m += 32) fn(S.cand[m]);
        },
        cmin, cmax, &need, S.hist);
    if (few) {
      // 4. the evicted positions as a bitmap over the row (hist, 128 words):
      // candidates below T, and ties past the first `need`
      uint32_t* evb = S.hist;
      __syncwarp();                                // the radix search is done with hist
      reinterpret_cast<uint4*>(evb)[lane] = make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
      uint32_t ties = 0;
      for (int m0 = 0; m0 < nc; m0 += 32) {
        const int m = m0 + lane;
        const uint32_t k = m < nc ? S.cand[m] : 0xffffffffu;
        const bool tie = m < nc && k == T;
        const uint32_t tm = __ballot_sync(0xffffffffu, tie);
        if (m < nc && (k < T || (tie && ties + __popc(tm & lt) >= need))) {
          const int i = S.cidx[m];
          atomicOr(&evb[i >> 5], 1u << (i & 31));
        }
        ties += __popc(tm);
      }
      __syncwarp();
      // evicted positions before each word (lane l owns words 4 l .. 4 l + 3),
      // in the second half of hist
      const uint4 wv = reinterpret_cast<const uint4*>(evb)[lane];
      const uint32_t c0 = __popc(wv.x), c1 = __popc(wv.y), c2 = __popc(wv.z), c3 = __popc(wv.w);
      const uint32_t mine = c0 + c1 + c2 + c3;
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t ex = incl - mine;
      __syncwarp();                                // every lane has read its candidates
      reinterpret_cast<uint4*>(S.hist + 128)[lane] = make_uint4(ex, ex + c0, ex + c0 + c1, ex + c0 + c1 + c2);
      __syncwarp();
      const uint32_t evicted = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) TRI_CHECK(evicted == static_cast<uint32_t>(n - B));      // exactly B kept
      (void)evicted;
      // kept position p goes to slot p - #{evicted before p}: each lane takes
      // 4 consecutive positions of a 128-position chunk (one bitmap word)
      const uint32_t* ebw = S.hist + 128;
      const int sh = (4 * lane) & 31;
      for (int j = 0; j < chunks; ++j) {
        const int p0 = 128 * j + 4 * lane;
        const int w = p0 >> 5;
        const uint32_t bits = evb[w];
        uint32_t e = ebw[w] + __popc(bits & ((1u << sh) - 1u));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t ev = (bits >> (sh + q)) & 1u;
          const int slot = p0 + q - static_cast<int>(e);
          if (!ev && p0 + q < n && slot < B) kept[slot] = p0 + q;     // slot < B unless the count is off
          e += ev;
        }
      }
      return true;
    }
  } else {
    // whole-row search: every key of the row counts (NaN keys are 0, below
    // every t >= 1 the search tests)
    auto each_key = [&](auto fn) {
      for (int j = 0; j < chunks; ++j) {
        const float4 xv = row_chunk(row, n, full, j, lane);
        const float v[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (valid(j, q)) fn(order_key(v[q]));
      }
    };
    need = static_cast<uint32_t>(B);
    T = warp_radix_kth(each_key, 0u, 0xffffffffu, &need, S.hist);
  }

  // 4'. T is the B-th largest key; keep every key above it and the `need`
  // lowest-index keys equal to it.  Emit in index order, comparing floats:
  // above T means a greater float (every number, if T is NaN's key), equal
  // to T a float that compares equal (NaN, if T is NaN's key).
  const bool t_nan = T == 0u;
  const float tf = key_value(T);
  uint32_t slot = 0, ties = 0;
  for (int j = 0; j < chunks; ++j) {
    const float4 xv = row_chunk(row, n, full, j, lane);
    const float v[4] = {xv.x, xv.y, xv.z, xv.w};
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
  return false;
}

// The in-place hole fill of a row from the bitmap of its evicted positions
// (evb, with ebw[w] the evicted positions before word w; n - B of them):
// the evicted positions below B are the holes, the kept positions at or
// above B the movers, and the r-th mover goes to the r-th hole -- the same
// moves as compact::holefill_unit_warp, found without reading the kept list
// back.  The holes are listed in `holes` (n - B ints of shared memory), in
// order.  The tail [B, n) is taken kFillChunk positions at a time: every lane
// ranks the movers among its 4 positions and computes their source and
// destination offsets (for a paged cache all the chunk's page lookups are in
// flight at once) into `offs` (2 x kFillChunk int64 of shared memory); then
// the chunk's rows are copied kFillBatch at a time, one 16-byte load per
// lane and row (lanes 0-15 K, 16-31 V), all loads in flight before the stores.
constexpr int kFillChunk = 128;
constexpr int kFillBatch = 8;

__device__ __forceinline__ void warp_fill_row(const Geom& g, int l, int h, int b, const uint32_t* evb,
                                              const uint32_t* ebw, int B, int n, int32_t* holes, int64_t* offs,
                                              uint16_t* k, uint16_t* v) {
  const int lane = threadIdx.x & 31, l16 = lane & 15, hw = lane >> 4;
  const int wb = B >> 5, sb = B & 31;
  const int m = static_cast<int>(ebw[wb] + __popc(evb[wb] & ((1u << sb) - 1u)));   // holes below B
  for (int w = lane; w < wb + (sb != 0); w += 32) {
    uint32_t bits = evb[w];
    if (w == wb) bits &= (1u << sb) - 1u;          // the word that straddles B
    uint32_t idx = ebw[w];
    while (bits) {
      holes[idx++] = 32 * w + __ffs(bits) - 1;
      bits &= bits - 1u;
    }
  }
  int64_t* const src = offs;                       // [kFillChunk] the chunk's movers, in mover order
  int64_t* const dst = offs + kFillChunk;          // [kFillChunk] their holes
  uint16_t* const base = hw ? v : k;
  int r0 = 0;                                      // movers of the chunks before
  for (int c0 = B; c0 < n; c0 += kFillChunk) {
    __syncwarp();                                  // the holes, or the previous chunk's copies, are done
    int slot[4], pos[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int p = c0 + 4 * lane + q;
      slot[q] = -1;
      pos[q] = p;
      if (p < n) {
        const uint32_t bits = evb[p >> 5];
        // kept positions in [B, p): (p - B) minus the evicted ones
        const int r = (p - B) - (static_cast<int>(ebw[p >> 5] + __popc(bits & ((1u << (p & 31)) - 1u))) - m);
        // r < m and r - r0 < kFillChunk unless the counts are off
        if (((bits >> (p & 31)) & 1u) == 0u && r < m && r - r0 < kFillChunk) slot[q] = r - r0;
      }
    }
    int64_t es[4], ed[4];
    bool ok[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {                  // every lookup of the lane before any is used
      ok[q] = slot[q] >= 0;
      if (ok[q]) {
        es[q] = row_elem(g, l, h, b, pos[q], &ok[q]);
        ed[q] = row_elem(g, l, h, b, holes[r0 + slot[q]], &ok[q]);
      }
    }
    int mine = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (slot[q] < 0) continue;
      ++mine;
      if (!ok[q]) flag(TRI_DEVFLAG_BAD_PAGE);
      src[slot[q]] = ok[q] ? es[q] : -1;
      dst[slot[q]] = ed[q];
    }
    const int mc = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(mine)));
    __syncwarp();
    for (int i0 = 0; i0 < mc; i0 += kFillBatch) {
      uint4 x[kFillBatch];
#pragma unroll
      for (int t = 0; t < kFillBatch; ++t) {
        const int64_t e = i0 + t < mc ? src[i0 + t] : -1;
        if (e >= 0) x[t] = ld_nc_v4(base + e + l16 * 8);
      }
#pragma unroll
      for (int t = 0; t < kFillBatch; ++t) {
        if (i0 + t < mc && src[i0 + t] >= 0) reinterpret_cast<uint4*>(base + dst[i0 + t])[l16] = x[t];
      }
    }
    r0 += mc;
  }
  if (lane == 0) TRI_CHECK(r0 == m);               // as many movers as holes
}

// One warp per unit, units [blockIdx.x * kWarpRows, ...): rows of at most
// kWarpMaxRow keys.  Dynamic shared memory: kWarpSmemBytes.  FILL: the
// in-place hole fill of each row follows its selection in the same warp
// (k, v: the cache), for launches whose rows move few keys.
template <bool FILL>
__global__ void __launch_bounds__(kWarpThreads, kWarpCtasPerSm) select_warp_kernel(const __grid_constant__ Geom g, const Args a,
                                                                   int units, uint16_t* k, uint16_t* v) {
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
  const bool bitmap = warp_select_row(a.scores + static_cast<int64_t>(u) * g.score_stride, n, B, scratch[w], kept);
  if constexpr (FILL) {
    int l, h, b_;
    compact::unit_coords(g, u, &l, &h, &b_);       // b_ == b
    __syncwarp();                                  // the kept list (global) and the bitmap (shared)
    if (bitmap && n - B <= kWarpCand)
      warp_fill_row(g, l, h, b, scratch[w].hist, scratch[w].hist + 128, B, n, scratch[w].cidx,
                    reinterpret_cast<int64_t*>(scratch[w].cand), k, v);
    else
      compact::holefill_unit_warp(g, kept, B, n, l, h, b, k, v);
  }
}

}  // namespace select
}  // namespace tri
