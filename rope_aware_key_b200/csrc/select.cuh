// Keep-highest selection: per unit, the top min(B, n) keys under the order
// (score descending, index ascending), written as ascending indices.
//
// Page "The future-offset average in TriAttention can be precomputed",
// opening section: the cache keeps its highest-scoring keys within a memory
// budget.  The budget B is TriAttention's KV budget (README, default 2048).
//
// One CTA per unit, on the unit's row of the score matrix (L2-resident right
// after scoring).  Every decision is made on an order-preserving uint32 key
// of the fp32 score (NaN -> 0, the lowest; -0 -> +0), so it is exact:
//  1. rows of up to kMaxCached scores are held in shared memory as keys
//     (longer rows are re-read from global memory each pass); min / max of
//     all keys and of the finite ones;
//  2. a histogram over kBins equal-width bins of the finite value range
//     (monotone in the key) finds the bin holding the B-th largest key; a
//     warp-parallel 32-ary search turns that bin into its key interval
//     [cmin, cmax];
//  3. one ballot pass writes a bitmap of the keys above cmax (all kept) and
//     collects the few keys inside [cmin, cmax] with their indices;
//  4. radix select (12-bit digits) over that short list gives the threshold
//     T, the B-th largest key, and `need`, how many keys equal to T are kept;
//     keys above T join the bitmap, keys equal to T go to a second bitmap of
//     which only the `need` lowest indices are kept;
//  5. the kept bitmap is written out in index order (popcounts, one block
//     scan), so the output is ascending and never depends on the order of
//     atomics.
// When the candidate list would overflow (heavy duplication), step 4 runs
// the radix over all keys instead and step 3 is redone against T.
#pragma once

#include "common.cuh"

namespace tri {
namespace select {

constexpr int kDigitBits = 12;
constexpr int kBins = 1 << kDigitBits;
constexpr int kMaxCached = 45056;          // keys held in shared memory (176 KB)
constexpr int kMaxLen = 655360;            // longest row (its two bitmaps must fit in shared memory)
constexpr int kMaxCand = 2048;             // candidate list capacity
constexpr uint32_t kKeyNegInf = 0x007fffffu;
constexpr uint32_t kKeyPosInf = 0xff800000u;

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (s != s) return 0u;               // NaN ranks lowest
  if (u == 0x80000000u) u = 0u;        // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Value bin of a key: equal-width bins over [lo, lo + kBins/scale]; keys
// below lo (NaN, -inf) go to bin 0, +inf (and the unused patterns above it)
// to the last bin.  Non-decreasing over all 2^32 keys.
__device__ __forceinline__ int value_bin(uint32_t key, float lo, float scale) {
  if (key >= kKeyPosInf) return kBins - 1;
  const float v = key_value(key);
  if (!(v >= lo)) return 0;
  const float t = (v - lo) * scale;
  return t < static_cast<float>(kBins) ? static_cast<int>(t) : kBins - 1;
}

// Warp-collective: the smallest key k with value_bin(k) >= target, or 2^32.
__device__ __forceinline__ uint64_t first_key_in_bin(int target, float lo, float scale) {
  const int lane = threadIdx.x & 31;
  uint64_t a = 0, b = uint64_t{1} << 32;       // the answer lies in [a, b]; b == 2^32 means none
  while (a < b) {
    const uint64_t step = (b - a + 31) / 32;
    const uint64_t x = a + static_cast<uint64_t>(lane) * step;
    const bool valid = x < b;
    const bool p = valid ? value_bin(static_cast<uint32_t>(x), lo, scale) >= target : true;
    const uint32_t m = __ballot_sync(0xffffffffu, p);
    if (m == 0u) {                             // every probe below: answer after the last one
      a = a + 31 * step + 1;
      continue;
    }
    const int f = __ffs(m) - 1;
    if (f == 0) {
      b = a;                                   // P(a) holds
    } else {
      const uint64_t xf = a + static_cast<uint64_t>(f) * step;
      const uint64_t na = a + static_cast<uint64_t>(f - 1) * step + 1;
      b = xf < b ? xf : b;
      a = na;
    }
  }
  return a;
}

struct Args {
  const float* scores;
  int32_t* kept;
  int32_t* kept_count;
  int B;
  int cap;          // >= every row length, a multiple of 4: sizes the shared-memory arrays
};

template <bool CACHED>
__device__ __forceinline__ uint32_t key_at(const float* __restrict__ row, const uint32_t* skeys, int i) {
  return CACHED ? skeys[i] : order_key(row[i]);
}

// Block-wide: find the digit d with (count above d) < need <= (count above d) + hist[d],
// scanning bins from the top.  Returns d; *above gets the count above d.
template <int NT>
__device__ __forceinline__ int find_digit(const uint32_t* hist, int nbins, uint32_t need, uint32_t* scan_sh,
                                          uint32_t* s_pair, uint32_t* above) {
  constexpr int kPer = (kBins + NT - 1) / NT;     // thread j owns bins [nbins - kPer(j+1), nbins - kPer j)
  const int hi = nbins - kPer * static_cast<int>(threadIdx.x);
  const int lo = max(0, hi - kPer);
  uint32_t sum = 0;
  for (int i = lo; i < hi; ++i) sum += hist[i];
  uint32_t total;
  const uint32_t before = block_exclusive_sum<NT>(sum, scan_sh, &total);
  if (before < need && before + sum >= need) {
    uint32_t acc = before;
    int d = lo;
    for (int i = hi - 1; i >= lo; --i) {
      if (acc + hist[i] >= need) {
        d = i;
        break;
      }
      acc += hist[i];
    }
    s_pair[0] = static_cast<uint32_t>(d);
    s_pair[1] = acc;
  }
  __syncthreads();
  *above = s_pair[1];
  const int d = static_cast<int>(s_pair[0]);
  __syncthreads();
  return d;
}

template <int NT>
__device__ __forceinline__ void block_minmax4(uint32_t* v, uint32_t (*sh)[NT / 32]) {
  // v[0], v[2]: minima; v[1], v[3]: maxima
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v[0] = __reduce_min_sync(0xffffffffu, v[0]);
  v[1] = __reduce_max_sync(0xffffffffu, v[1]);
  v[2] = __reduce_min_sync(0xffffffffu, v[2]);
  v[3] = __reduce_max_sync(0xffffffffu, v[3]);
  if (lane == 0)
    for (int j = 0; j < 4; ++j) sh[j][warp] = v[j];
  __syncthreads();
  if (warp == 0) {
    uint32_t x[4];
    x[0] = lane < NT / 32 ? sh[0][lane] : 0xffffffffu;
    x[1] = lane < NT / 32 ? sh[1][lane] : 0u;
    x[2] = lane < NT / 32 ? sh[2][lane] : 0xffffffffu;
    x[3] = lane < NT / 32 ? sh[3][lane] : 0u;
    x[0] = __reduce_min_sync(0xffffffffu, x[0]);
    x[1] = __reduce_max_sync(0xffffffffu, x[1]);
    x[2] = __reduce_min_sync(0xffffffffu, x[2]);
    x[3] = __reduce_max_sync(0xffffffffu, x[3]);
    if (lane == 0)
      for (int j = 0; j < 4; ++j) sh[j][0] = x[j];
  }
  __syncthreads();
  for (int j = 0; j < 4; ++j) v[j] = sh[j][0];
  __syncthreads();
}

// Radix search for the need-th largest key among those for which
// `visit(fn)` calls fn(key) (the candidates).  Returns T; *need becomes the
// number of keys equal to T to keep.  `lo_key`..`hi_key` bound the candidates.
template <int NT, typename Visit>
__device__ __forceinline__ uint32_t radix_threshold(Visit visit, uint32_t lo_key, uint32_t hi_key, uint32_t* need,
                                                    uint32_t* hist, uint32_t* scan_sh, uint32_t* s_pair) {
  if (lo_key == hi_key) return hi_key;
  int known = __clz(lo_key ^ hi_key);
  uint32_t prefix = known ? (hi_key & (0xffffffffu << (32 - known))) : 0u;
  while (known < 32) {
    const int bits = min(kDigitBits, 32 - known);
    const int shift = 32 - known - bits;
    const int nbins = 1 << bits;
    for (int i = threadIdx.x; i < nbins; i += NT) hist[i] = 0;
    __syncthreads();
    const uint32_t pfx = prefix;
    const int kn = known;
    visit([&](uint32_t key) {
      if (kn == 0 || ((key ^ pfx) >> (32 - kn)) == 0u) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
    });
    __syncthreads();
    uint32_t above;
    const int d = find_digit<NT>(hist, nbins, *need, scan_sh, s_pair, &above);
    prefix |= static_cast<uint32_t>(d) << shift;
    *need -= above;
    known += bits;
  }
  return prefix;
}

template <int NT, bool CACHED>
__global__ void __launch_bounds__(NT) select_kernel(const __grid_constant__ Geom g, const Args a) {
  constexpr int NW = NT / 32;
  extern __shared__ uint4 select_dyn[];
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t scan_sh[NW];
  __shared__ uint32_t red[4][NW];
  __shared__ uint32_t s_pair[2];
  __shared__ uint32_t s_bounds[2];
  __shared__ uint32_t s_ncand;

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

  // dynamic shared memory: [keys (CACHED)] [kept bitmap] [tie bitmap] [candidate keys] [candidate indices]
  const int cap = a.cap;
  const int words = (n + 31) >> 5;
  const int wcap = (cap + 31) >> 5;
  uint32_t* skeys = reinterpret_cast<uint32_t*>(select_dyn);
  uint32_t* keepmap = skeys + (CACHED ? cap : 0);
  uint32_t* tiemap = keepmap + wcap;
  uint32_t* cand_key = tiemap + wcap;
  int32_t* cand_idx = reinterpret_cast<int32_t*>(cand_key + kMaxCand);

  // ---- 1. keys, min / max of all keys and of the finite ones
  uint32_t mm[4] = {0xffffffffu, 0u, 0xffffffffu, 0u};
  for (int i = threadIdx.x * 4; i < n; i += NT * 4) {
    uint32_t t[4];
    if (i + 3 < n) {
      const float4 v = *reinterpret_cast<const float4*>(row + i);
      t[0] = order_key(v.x); t[1] = order_key(v.y); t[2] = order_key(v.z); t[3] = order_key(v.w);
      if (CACHED) *reinterpret_cast<uint4*>(skeys + i) = make_uint4(t[0], t[1], t[2], t[3]);
    } else {
      for (int e = 0; e < 4; ++e) {
        t[e] = i + e < n ? order_key(row[i + e]) : 0u;
        if (CACHED && i + e < n) skeys[i + e] = t[e];
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i + e < n) {
        mm[0] = min(mm[0], t[e]);
        mm[1] = max(mm[1], t[e]);
        if (t[e] > kKeyNegInf && t[e] < kKeyPosInf) {
          mm[2] = min(mm[2], t[e]);
          mm[3] = max(mm[3], t[e]);
        }
      }
    }
  }
  for (int w = threadIdx.x; w < words; w += NT) tiemap[w] = 0u;
  if (threadIdx.x == 0) s_ncand = 0;
  block_minmax4<NT>(mm, red);
  const uint32_t kmin = mm[0], kmax = mm[1];

  if (kmin == kmax) {                          // all scores equal: the B lowest indices
    for (int j = threadIdx.x; j < B; j += NT) kept[j] = j;
    return;
  }

  // ---- 2. the bin of the B-th largest key and its key interval
  uint32_t need = static_cast<uint32_t>(B);   // still to take inside [cmin, cmax]
  uint32_t cmin = kmin, cmax = kmax;
  uint32_t ncand_expected = static_cast<uint32_t>(n);
  float lo = 0.f, scale = 0.f;
  bool binned = false;
  if (mm[2] < mm[3]) {
    lo = key_value(mm[2]);
    const float width = key_value(mm[3]) - lo;
    scale = static_cast<float>(kBins) / width;
    binned = width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f;
  }
  if (binned) {
    for (int i = threadIdx.x; i < kBins; i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) atomicAdd(&hist[value_bin(key_at<CACHED>(row, skeys, i), lo, scale)], 1u);
    __syncthreads();
    uint32_t above;
    const int bin = find_digit<NT>(hist, kBins, need, scan_sh, s_pair, &above);
    need -= above;
    ncand_expected = hist[bin];
    if (warp == 0) {
      const uint64_t k0 = first_key_in_bin(bin, lo, scale);
      const uint64_t k1 = bin + 1 < kBins ? first_key_in_bin(bin + 1, lo, scale) : (uint64_t{1} << 32);
      if (lane == 0) {
        s_bounds[0] = static_cast<uint32_t>(k0);
        s_bounds[1] = static_cast<uint32_t>(k1 - 1);
      }
    }
    __syncthreads();
    cmin = s_bounds[0];
    cmax = s_bounds[1];
  }
  const bool listed = ncand_expected <= static_cast<uint32_t>(kMaxCand);

  // ---- 3. bitmap of the keys above cmax; candidates in [cmin, cmax]
  for (int base = warp * 32; base < n; base += NT) {
    const int i = base + lane;
    const uint32_t k = i < n ? key_at<CACHED>(row, skeys, i) : 0u;
    const bool in = i < n;
    const uint32_t m = __ballot_sync(0xffffffffu, in && k > cmax);
    if (lane == 0) keepmap[base >> 5] = m;
    if (listed && in && k >= cmin && k <= cmax) {
      const uint32_t pos = atomicAdd(&s_ncand, 1u);
      cand_key[pos] = k;
      cand_idx[pos] = i;
    }
  }
  __syncthreads();

  // ---- 4. threshold among the candidates, then mark them
  if (listed) {
    const int nc = static_cast<int>(s_ncand);
    const uint32_t T = radix_threshold<NT>(
        [&](auto fn) {
          for (int j = threadIdx.x; j < nc; j += NT) fn(cand_key[j]);
        },
        cmin, cmax, &need, hist, scan_sh, s_pair);
    for (int j = threadIdx.x; j < nc; j += NT) {
      const uint32_t k = cand_key[j];
      const int i = cand_idx[j];
      if (k > T) atomicOr(&keepmap[i >> 5], 1u << (i & 31));
      else if (k == T) atomicOr(&tiemap[i >> 5], 1u << (i & 31));
    }
  } else {
    const uint32_t T = radix_threshold<NT>(
        [&](auto fn) {
          for (int i = threadIdx.x; i < n; i += NT) {
            const uint32_t k = key_at<CACHED>(row, skeys, i);
            if (k >= cmin && k <= cmax) fn(k);
          }
        },
        cmin, cmax, &need, hist, scan_sh, s_pair);
    for (int base = warp * 32; base < n; base += NT) {
      const int i = base + lane;
      const uint32_t k = i < n ? key_at<CACHED>(row, skeys, i) : 0u;
      const uint32_t mk = __ballot_sync(0xffffffffu, i < n && k > T);
      const uint32_t mt = __ballot_sync(0xffffffffu, i < n && k == T);
      if (lane == 0) {
        keepmap[base >> 5] = mk;
        tiemap[base >> 5] = mt;
      }
    }
  }
  __syncthreads();

  // ---- 5. ties: keep the `need` lowest indices equal to T; then write out
  const int per = (words + NT - 1) / NT;              // words per thread, contiguous
  const int w0 = min(words, static_cast<int>(threadIdx.x) * per);
  const int w1 = min(words, w0 + per);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(tiemap[w]);
  uint32_t total;
  uint32_t before = block_exclusive_sum<NT>(cnt, scan_sh, &total);
  for (int w = w0; w < w1 && before < need; ++w) {
    uint32_t m = tiemap[w], take = 0u;
    while (m && before < need) {
      const uint32_t bit = m & (~m + 1u);
      take |= bit;
      m ^= bit;
      ++before;
    }
    if (take) keepmap[w] |= take;
  }
  __syncthreads();
  cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(keepmap[w]);
  uint32_t slot = block_exclusive_sum<NT>(cnt, scan_sh, &total);
  for (int w = w0; w < w1; ++w) {
    uint32_t m = keepmap[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      kept[slot++] = w * 32 + bit;
      m &= m - 1u;
    }
  }
}

// Dynamic shared memory of select_kernel for rows of `cap` floats.
inline size_t smem_bytes(int64_t cap, bool cached) {
  const int64_t wcap = (cap + 31) / 32;
  return static_cast<size_t>((cached ? cap : 0) + 2 * wcap + 2 * kMaxCand) * 4;
}

}  // namespace select
}  // namespace tri
