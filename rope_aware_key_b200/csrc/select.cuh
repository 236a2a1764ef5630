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
//  1. evenly spaced samples of the row give a key L such that, for any but a
//     pathological order of the scores, between B and lcap keys are >= L
//     (the sample's (B/n share + 5 sigma)-quantile, via a value histogram);
//  2. one pass lists every key >= L with its index (warp-aggregated appends
//     into shared memory);
//  3. radix select (11-bit digits) over the list gives the threshold T, the
//     B-th largest key, and `need`, how many keys equal to T are kept; kept
//     keys are marked in a bitmap, keys equal to T in a tie bitmap;
//  4. the `need` lowest-index ties join the bitmap, which is written out in
//     index order (popcounts, block scans): the output is ascending and never
//     depends on the order of atomics.
// If the count of keys >= L falls outside [B, lcap], an exact path over the
// whole row replaces steps 1-3: a value histogram finds the bin of the B-th
// largest key, a ballot pass marks everything above the bin and lists the
// bin's keys, and the radix runs on that list (or on the whole row if the
// bin is too crowded).
#pragma once

#include "common.cuh"

namespace tri {
namespace select {

constexpr int kDigitBits = 11;
constexpr int kBins = 1 << kDigitBits;
constexpr int kSamples = 4096;             // evenly spaced scores that bound the threshold
constexpr int kMaxShared = 200 * 1024;     // dynamic shared memory one CTA may use
constexpr uint32_t kKeyNegInf = 0x007fffffu;
constexpr uint32_t kKeyPosInf = 0xff800000u;

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  const bool nan = (u & 0x7fffffffu) > 0x7f800000u;      // NaN ranks lowest
  u = u == 0x80000000u ? 0u : u;                         // -0 ranks with +0
  const uint32_t k = u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
  return nan ? 0u : k;
}

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Value bin of a real key (one that order_key can produce): equal-width bins,
// bin = clamp(trunc(v * scale - lo_s), 0, kBins - 1).  The fused multiply-add
// and the saturating conversion are monotone, NaN converts to 0 and -inf / +inf
// saturate to the first / last bin, so the bin never decreases with the key.
__device__ __forceinline__ int value_bin(uint32_t key, float scale, float lo_s) {
  const int t = __float2int_rz(fmaf(key_value(key), scale, -lo_s));
  return min(max(t, 0), kBins - 1);
}

// The same over all 2^32 bit patterns (the unused ones above +inf's key go to
// the last bin), for the key-space search.
__device__ __forceinline__ int value_bin_any(uint32_t key, float scale, float lo_s) {
  return key >= kKeyPosInf ? kBins - 1 : value_bin(key, scale, lo_s);
}

// Warp-collective: the smallest key k with value_bin(k) >= target, or 2^32.
__device__ __forceinline__ uint64_t first_key_in_bin(int target, float scale, float lo_s) {
  const int lane = threadIdx.x & 31;
  uint64_t a = 0, b = uint64_t{1} << 32;       // the answer lies in [a, b]; b == 2^32 means none
  while (a < b) {
    const uint64_t step = (b - a + 31) / 32;
    const uint64_t x = a + static_cast<uint64_t>(lane) * step;
    const bool valid = x < b;
    const bool p = valid ? value_bin_any(static_cast<uint32_t>(x), scale, lo_s) >= target : true;
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
  int cap;          // >= every row length, a multiple of 4: sizes the shared-memory bitmaps
  int lcap;         // capacity of the shared-memory key list
};

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

// Shared-memory layout of one CTA (dynamic part), all 32-bit words:
//   list_key[max(lcap, kSamples)] list_idx[lcap] keepmap[wcap] tiemap[wcap];
// the samples live in list_key until the list is filled.
struct Smem {
  uint32_t* list_key;
  int32_t* list_idx;
  uint32_t* keepmap;
  uint32_t* tiemap;
  uint32_t* samples;
};

// Exact threshold over the whole row (read from global memory): value-bin
// histogram, the bin's key interval, a ballot pass that writes the kept
// bitmap above the interval and lists the keys inside it, then radix select
// over that list (or over the whole row if the list would overflow).  Marks
// keys above T in keepmap and keys equal to T in tiemap; returns `need`, the
// number of ties to keep.
template <int NT>
__device__ __forceinline__ uint32_t exact_path(const float* __restrict__ row, int n, int B, int lcap, const Smem& m,
                                               uint32_t* hist, uint32_t* scan_sh, uint32_t (*red)[NT / 32],
                                               uint32_t* s_pair, uint32_t* s_bounds, uint32_t* s_count) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int words = (n + 31) >> 5;
  __syncthreads();                                 // the sampled path is done with the shared arrays
  // min / max of all keys and of the finite ones
  uint32_t mm[4] = {0xffffffffu, 0u, 0xffffffffu, 0u};
  for (int i = threadIdx.x; i < n; i += NT) {
    const uint32_t k = order_key(row[i]);
    mm[0] = min(mm[0], k);
    mm[1] = max(mm[1], k);
    if (k > kKeyNegInf && k < kKeyPosInf) {
      mm[2] = min(mm[2], k);
      mm[3] = max(mm[3], k);
    }
  }
  for (int w = threadIdx.x; w < words; w += NT) m.tiemap[w] = 0u;
  if (threadIdx.x == 0) *s_count = 0;
  block_minmax4<NT>(mm, red);
  uint32_t need = static_cast<uint32_t>(B);
  uint32_t cmin = mm[0], cmax = mm[1];
  uint32_t ncand = static_cast<uint32_t>(n);
  float scale = 0.f, lo_s = 0.f;
  bool binned = false;
  if (mm[2] < mm[3]) {
    const float lo = key_value(mm[2]);
    const float width = key_value(mm[3]) - lo;
    scale = static_cast<float>(kBins) / width;
    lo_s = lo * scale;
    binned = width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s);
  }
  if (binned) {
    for (int i = threadIdx.x; i < kBins; i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) atomicAdd(&hist[value_bin(order_key(row[i]), scale, lo_s)], 1u);
    __syncthreads();
    uint32_t above;
    const int bin = find_digit<NT>(hist, kBins, need, scan_sh, s_pair, &above);
    need -= above;
    ncand = hist[bin];
    if (warp == 0) {
      const uint64_t k0 = first_key_in_bin(bin, scale, lo_s);
      const uint64_t k1 = bin + 1 < kBins ? first_key_in_bin(bin + 1, scale, lo_s) : (uint64_t{1} << 32);
      if (lane == 0) {
        s_bounds[0] = static_cast<uint32_t>(k0);
        s_bounds[1] = static_cast<uint32_t>(k1 - 1);
      }
    }
    __syncthreads();
    cmin = s_bounds[0];
    cmax = s_bounds[1];
  }
  const bool listed = ncand <= static_cast<uint32_t>(lcap);
  for (int base = warp * 32; base < n; base += NT) {
    const int i = base + lane;
    const bool in = i < n;
    const uint32_t k = in ? order_key(row[i]) : 0u;
    const uint32_t bits = __ballot_sync(0xffffffffu, in && k > cmax);
    if (lane == 0) m.keepmap[base >> 5] = bits;
    if (listed && in && k >= cmin && k <= cmax) {
      const uint32_t pos = atomicAdd(s_count, 1u);
      m.list_key[pos] = k;
      m.list_idx[pos] = i;
    }
  }
  __syncthreads();
  if (listed) {
    const int nc = static_cast<int>(*s_count);
    const uint32_t T = radix_threshold<NT>(
        [&](auto fn) {
          for (int j = threadIdx.x; j < nc; j += NT) fn(m.list_key[j]);
        },
        cmin, cmax, &need, hist, scan_sh, s_pair);
    for (int j = threadIdx.x; j < nc; j += NT) {
      const uint32_t k = m.list_key[j];
      const int i = m.list_idx[j];
      if (k > T) atomicOr(&m.keepmap[i >> 5], 1u << (i & 31));
      else if (k == T) atomicOr(&m.tiemap[i >> 5], 1u << (i & 31));
    }
  } else {
    const uint32_t T = radix_threshold<NT>(
        [&](auto fn) {
          for (int i = threadIdx.x; i < n; i += NT) {
            const uint32_t k = order_key(row[i]);
            if (k >= cmin && k <= cmax) fn(k);
          }
        },
        cmin, cmax, &need, hist, scan_sh, s_pair);
    for (int base = warp * 32; base < n; base += NT) {
      const int i = base + lane;
      const uint32_t k = i < n ? order_key(row[i]) : 0u;
      const uint32_t mk = __ballot_sync(0xffffffffu, i < n && k > T);
      const uint32_t mt = __ballot_sync(0xffffffffu, i < n && k == T);
      if (lane == 0) {
        m.keepmap[base >> 5] = mk;
        m.tiemap[base >> 5] = mt;
      }
    }
  }
  __syncthreads();
  return need;
}

// Sampled path.  kSamples evenly spaced scores give a key L that at least
// `r` samples reach, r chosen well above the B/n share of the samples, so
// that (for any but a pathological order of the scores) between B and lcap
// keys of the row are >= L.  One pass lists exactly those keys; the B-th
// largest of the list is then the B-th largest of the row.  Returns false
// (having written nothing) when the count falls outside [B, lcap].
template <int NT>
__device__ __forceinline__ bool sampled_path(const float* __restrict__ row, int n, int B, int lcap, const Smem& m,
                                             uint32_t* hist, uint32_t* scan_sh, uint32_t (*red)[NT / 32],
                                             uint32_t* s_pair, uint32_t* s_bounds, uint32_t* s_count,
                                             uint32_t* need_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int words = (n + 31) >> 5;
  const int ms = min(n, kSamples);
  uint32_t mm[4] = {0xffffffffu, 0u, 0xffffffffu, 0u};
  for (int j = threadIdx.x; j < ms; j += NT) {
    const int i = static_cast<int>(static_cast<int64_t>(j) * n / ms);
    const uint32_t k = order_key(row[i]);
    m.samples[j] = k;
    if (k > kKeyNegInf && k < kKeyPosInf) {
      mm[2] = min(mm[2], k);
      mm[3] = max(mm[3], k);
    }
  }
  for (int w = threadIdx.x; w < words; w += NT) {
    m.keepmap[w] = 0u;
    m.tiemap[w] = 0u;
  }
  if (threadIdx.x == 0) *s_count = 0;
  block_minmax4<NT>(mm, red);
  const float qm = static_cast<float>(B) * static_cast<float>(ms) / static_cast<float>(n);
  const int r = static_cast<int>(ceilf(qm + 5.f * sqrtf(qm) + 20.f));
  uint32_t L = 0u;                                 // r >= ms: every key is listed
  if (r < ms) {
    if (!(mm[2] < mm[3])) return false;            // no spread among the samples
    const float lo = key_value(mm[2]);
    const float width = key_value(mm[3]) - lo;
    const float scale = static_cast<float>(kBins) / width;
    const float lo_s = lo * scale;
    if (!(width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s))) return false;
    for (int i = threadIdx.x; i < kBins; i += NT) hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < ms; j += NT) atomicAdd(&hist[value_bin(m.samples[j], scale, lo_s)], 1u);
    __syncthreads();
    uint32_t above;
    const int bin = find_digit<NT>(hist, kBins, static_cast<uint32_t>(r), scan_sh, s_pair, &above);
    if (warp == 0) {
      const uint64_t k0 = first_key_in_bin(bin, scale, lo_s);
      if (lane == 0) s_bounds[0] = static_cast<uint32_t>(k0);
    }
    __syncthreads();
    L = s_bounds[0];
  }
  // list every key >= L (warp-aggregated appends)
  uint32_t lmax = 0u;
  for (int base = warp * 128; base < n; base += NT * 4) {
    const int i = base + lane * 4;
    uint32_t k[4];
    if (i + 3 < n) {
      const float4 v = *reinterpret_cast<const float4*>(row + i);
      k[0] = order_key(v.x); k[1] = order_key(v.y); k[2] = order_key(v.z); k[3] = order_key(v.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) k[e] = i + e < n ? order_key(row[i + e]) : 0u;
    }
    uint32_t flags = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool f = i + e < n && k[e] >= L;
      flags |= static_cast<uint32_t>(f) << e;
      lmax = f ? max(lmax, k[e]) : lmax;
    }
    const uint32_t c = __popc(flags);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t pos = 0;
    if (lane == 0 && total) pos = atomicAdd(s_count, total);
    pos = __shfl_sync(0xffffffffu, pos, 0) + incl - c;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (flags & (1u << e)) {
        if (pos < static_cast<uint32_t>(lcap)) {
          m.list_key[pos] = k[e];
          m.list_idx[pos] = i + e;
        }
        ++pos;
      }
    }
  }
  lmax = __reduce_max_sync(0xffffffffu, lmax);
  if (lane == 0) red[1][warp] = lmax;
  __syncthreads();
  const uint32_t c = *s_count;
  const bool ok = c >= static_cast<uint32_t>(B) && c <= static_cast<uint32_t>(lcap);
  __syncthreads();                                 // every thread has read s_count
  if (!ok) return false;
  uint32_t hi = 0u;
  for (int w = 0; w < NT / 32; ++w) hi = max(hi, red[1][w]);
  __syncthreads();
  uint32_t need = static_cast<uint32_t>(B);
  const int nc = static_cast<int>(c);
  const uint32_t T = radix_threshold<NT>(
      [&](auto fn) {
        for (int j = threadIdx.x; j < nc; j += NT) fn(m.list_key[j]);
      },
      L, hi, &need, hist, scan_sh, s_pair);
  for (int j = threadIdx.x; j < nc; j += NT) {
    const uint32_t k = m.list_key[j];
    const int i = m.list_idx[j];
    if (k > T) atomicOr(&m.keepmap[i >> 5], 1u << (i & 31));
    else if (k == T) atomicOr(&m.tiemap[i >> 5], 1u << (i & 31));
  }
  __syncthreads();
  *need_out = need;
  return true;
}

template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(const __grid_constant__ Geom g, const Args a) {
  constexpr int NW = NT / 32;
  extern __shared__ uint4 select_dyn[];
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t scan_sh[NW];
  __shared__ uint32_t red[4][NW];
  __shared__ uint32_t s_pair[2];
  __shared__ uint32_t s_bounds[2];
  __shared__ uint32_t s_count;

  const int u = blockIdx.x;
  const int b = u % g.batch;
  const int n = g.len[b];
  const int B = a.B;
  const float* __restrict__ row = a.scores + static_cast<int64_t>(u) * g.score_stride;
  int32_t* __restrict__ kept = a.kept + static_cast<int64_t>(u) * B;

  if (threadIdx.x == 0) a.kept_count[u] = min(n, B);
  if (n <= B) {
    for (int i = threadIdx.x; i < n; i += NT) kept[i] = i;
    return;
  }

  const int wcap = (a.cap + 31) >> 5;
  Smem m;
  m.list_key = reinterpret_cast<uint32_t*>(select_dyn);
  m.samples = m.list_key;
  m.list_idx = reinterpret_cast<int32_t*>(m.list_key + max(a.lcap, kSamples));
  m.keepmap = reinterpret_cast<uint32_t*>(m.list_idx + a.lcap);
  m.tiemap = m.keepmap + wcap;

  uint32_t need;
  if (!sampled_path<NT>(row, n, B, a.lcap, m, hist, scan_sh, red, s_pair, s_bounds, &s_count, &need))
    need = exact_path<NT>(row, n, B, a.lcap, m, hist, scan_sh, red, s_pair, s_bounds, &s_count);

  // ties: keep the `need` lowest indices equal to T; then write out in index order
  const int words = (n + 31) >> 5;
  const int per = (words + NT - 1) / NT;              // words per thread, contiguous
  const int w0 = min(words, static_cast<int>(threadIdx.x) * per);
  const int w1 = min(words, w0 + per);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(m.tiemap[w]);
  uint32_t total;
  uint32_t before = block_exclusive_sum<NT>(cnt, scan_sh, &total);
  for (int w = w0; w < w1 && before < need; ++w) {
    uint32_t bits = m.tiemap[w], take = 0u;
    while (bits && before < need) {
      const uint32_t bit = bits & (~bits + 1u);
      take |= bit;
      bits ^= bit;
      ++before;
    }
    if (take) m.keepmap[w] |= take;
  }
  __syncthreads();
  cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(m.keepmap[w]);
  uint32_t slot = block_exclusive_sum<NT>(cnt, scan_sh, &total);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = m.keepmap[w];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      kept[slot++] = w * 32 + bit;
      bits &= bits - 1u;
    }
  }
}

// Capacity of the key list for budget B on rows of at most `cap` keys.
inline int list_capacity(int B, int cap) {
  const int64_t want = int64_t{B} + B / 2 + 2048;
  return static_cast<int>(want < cap ? want : cap);
}

// Dynamic shared memory of select_kernel.
inline size_t smem_bytes(int cap, int lcap) {
  const int64_t wcap = (int64_t{cap} + 31) / 32;
  const int64_t keys = lcap > kSamples ? lcap : kSamples;
  return static_cast<size_t>(keys + int64_t{lcap} + 2 * wcap) * 4;
}

}  // namespace select
}  // namespace tri
