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

// Warp-collective: the smallest key k with value_bin(k) >= target, or 2^32,
// by a 32-ary search over the key space.
__device__ __forceinline__ uint64_t first_key_search(int target, float scale, float lo_s) {
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

// The same, first trying the 32 keys around the value where the bin starts
// ((target + lo_s) / scale): if the bin boundary falls among them, one
// ballot finds it; otherwise the full search runs.  Warp-collective.
__device__ __forceinline__ uint64_t first_key_in_bin(int target, float scale, float lo_s) {
  const int lane = threadIdx.x & 31;
  const float v = (static_cast<float>(target) + lo_s) / scale;
  if (target > 0 && target < kBins && isfinite(v)) {
    const uint32_t g = order_key(v);
    if (g >= 16u && g < 0xffffffffu - 16u) {
      const uint32_t x = g - 16u + static_cast<uint32_t>(lane);
      const uint32_t m = __ballot_sync(0xffffffffu, value_bin_any(x, scale, lo_s) >= target);
      if (m != 0u && (m & 1u) == 0u) return g - 16u + static_cast<uint32_t>(__ffs(m) - 1);
    }
  }
  return first_key_search(target, scale, lo_s);
}

struct Args {
  const float* scores;
  int32_t* kept;
  int32_t* kept_count;
  int B;
  int cap;          // >= every row length, a multiple of 4: sizes the shared-memory bitmaps
  int lcap;         // capacity of the shared-memory key list
};

// A group of NT threads that selects one row: the whole CTA (BAR == 0,
// synchronised by __syncthreads), or the warps [BASE/32, (BASE+NT)/32) of a
// larger CTA, synchronised by the named barrier BAR.
template <int NT_, int BASE_, int BAR_>
struct Group {
  static constexpr int NT = NT_;
  static constexpr int NW = NT_ / 32;
  static_assert(NT_ % 32 == 0 && BASE_ % 32 == 0, "whole warps");
  __device__ __forceinline__ static int tid() { return static_cast<int>(threadIdx.x) - BASE_; }
  __device__ __forceinline__ static int warp() { return tid() >> 5; }
  __device__ __forceinline__ static void sync() {
    if (BAR_ == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"n"(BAR_), "n"(NT_) : "memory");
  }
};

// Per-group shared scratch (static part).
template <class G>
struct Scratch {
  uint32_t hist[kBins];
  uint32_t scan[G::NW];
  uint32_t red[4][G::NW];
  uint32_t pair[2];
  uint32_t bounds[2];
  uint32_t count;
  uint32_t small[256];     // keys of one value bin (list_threshold)
};

// Dynamic shared-memory arrays of one row's selection, all 32-bit words:
//   list_key[max(lcap, kSamples)] list_idx[lcap] keepmap[wcap] tiemap[wcap];
// the samples live in list_key until the list is filled.
struct Smem {
  uint32_t* list_key;
  int32_t* list_idx;
  uint32_t* keepmap;
  uint32_t* tiemap;
  uint32_t* samples;
};

__device__ __forceinline__ Smem carve(uint32_t* base, int cap, int lcap) {
  Smem m;
  const int wcap = (cap + 31) >> 5;
  m.list_key = base;
  m.samples = base;
  m.list_idx = reinterpret_cast<int32_t*>(base + max(lcap, kSamples));
  m.keepmap = reinterpret_cast<uint32_t*>(m.list_idx + lcap);
  m.tiemap = m.keepmap + wcap;
  return m;
}

// Scores are read at L2 (ld.global.cg): in the fused kernel they were written
// by other SMs during the same launch.
__device__ __forceinline__ uint32_t key_at(const float* row, int i) { return order_key(__ldcg(row + i)); }

// In a TRI_CHECKED build: the first `nbins` bins of hist total `want`
// (every listed key landed in exactly one bin).  Call from the whole group.
template <class G>
__device__ __forceinline__ void check_hist_total(const uint32_t* hist, int nbins, uint32_t want, uint32_t* scan);

// Exclusive sum of v over the group; *total gets the group's sum.
template <class G>
__device__ __forceinline__ uint32_t group_exclusive_sum(uint32_t v, uint32_t* sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = G::warp();
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  G::sync();
  if (warp == 0) {
    uint32_t t = lane < G::NW ? sh[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < G::NW) sh[lane] = t;
  }
  G::sync();
  const uint32_t before = warp ? sh[warp - 1] : 0u;
  *total = sh[G::NW - 1];
  G::sync();
  return before + x - v;
}

template <class G>
__device__ __forceinline__ void check_hist_total(const uint32_t* hist, int nbins, uint32_t want, uint32_t* scan) {
#ifdef TRI_CHECKED
  uint32_t part = 0, total = 0;
  for (int i = G::tid(); i < nbins; i += G::NT) part += hist[i];
  group_exclusive_sum<G>(part, scan, &total);
  if (G::tid() == 0) TRI_CHECK(total == want);
#else
  (void)hist, (void)nbins, (void)want, (void)scan;
#endif
}

// The digit d with (count above d) < need <= (count above d) + hist[d],
// scanning bins from the top.  Returns d; *above gets the count above d.
template <class G>
__device__ __forceinline__ int find_digit(const uint32_t* hist, int nbins, uint32_t need, Scratch<G>& S,
                                          uint32_t* above) {
  constexpr int kPer = (kBins + G::NT - 1) / G::NT;   // thread j owns bins [nbins - kPer(j+1), nbins - kPer j)
  const int hi = nbins - kPer * G::tid();
  const int lo = max(0, hi - kPer);
  uint32_t sum = 0;
  for (int i = lo; i < hi; ++i) sum += hist[i];
  uint32_t total;
  const uint32_t before = group_exclusive_sum<G>(sum, S.scan, &total);
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
    S.pair[0] = static_cast<uint32_t>(d);
    S.pair[1] = acc;
  }
  G::sync();
  *above = S.pair[1];
  const int d = static_cast<int>(S.pair[0]);
  G::sync();
  return d;
}

// v[0], v[2] become group minima, v[1], v[3] group maxima.
template <class G>
__device__ __forceinline__ void group_minmax4(uint32_t* v, Scratch<G>& S) {
  const int lane = threadIdx.x & 31, warp = G::warp();
  v[0] = __reduce_min_sync(0xffffffffu, v[0]);
  v[1] = __reduce_max_sync(0xffffffffu, v[1]);
  v[2] = __reduce_min_sync(0xffffffffu, v[2]);
  v[3] = __reduce_max_sync(0xffffffffu, v[3]);
  if (lane == 0)
    for (int j = 0; j < 4; ++j) S.red[j][warp] = v[j];
  G::sync();
  if (warp == 0) {
    uint32_t x[4];
    x[0] = lane < G::NW ? S.red[0][lane] : 0xffffffffu;
    x[1] = lane < G::NW ? S.red[1][lane] : 0u;
    x[2] = lane < G::NW ? S.red[2][lane] : 0xffffffffu;
    x[3] = lane < G::NW ? S.red[3][lane] : 0u;
    x[0] = __reduce_min_sync(0xffffffffu, x[0]);
    x[1] = __reduce_max_sync(0xffffffffu, x[1]);
    x[2] = __reduce_min_sync(0xffffffffu, x[2]);
    x[3] = __reduce_max_sync(0xffffffffu, x[3]);
    if (lane == 0)
      for (int j = 0; j < 4; ++j) S.red[j][0] = x[j];
  }
  G::sync();
  for (int j = 0; j < 4; ++j) v[j] = S.red[j][0];
  G::sync();
}

// Radix search for the need-th largest key among those for which
// `visit(fn)` calls fn(key) (the candidates, all inside [lo_key, hi_key]).
// Returns T; *need becomes the number of keys equal to T to keep.
template <class G, typename Visit>
__device__ __forceinline__ uint32_t radix_threshold(Visit visit, uint32_t lo_key, uint32_t hi_key, uint32_t* need,
                                                    Scratch<G>& S) {
  if (lo_key == hi_key) return hi_key;
  int known = __clz(lo_key ^ hi_key);
  uint32_t prefix = known ? (hi_key & (0xffffffffu << (32 - known))) : 0u;
  while (known < 32) {
    const int bits = min(kDigitBits, 32 - known);
    const int shift = 32 - known - bits;
    const int nbins = 1 << bits;
    for (int i = G::tid(); i < nbins; i += G::NT) S.hist[i] = 0;
    G::sync();
    const uint32_t pfx = prefix;
    const int kn = known;
    visit([&](uint32_t key) {
      if (kn == 0 || ((key ^ pfx) >> (32 - kn)) == 0u) atomicAdd(&S.hist[(key >> shift) & (nbins - 1)], 1u);
    });
    G::sync();
    uint32_t above;
    const int d = find_digit<G>(S.hist, nbins, *need, S, &above);
    prefix |= static_cast<uint32_t>(d) << shift;
    *need -= above;
    known += bits;
  }
  return prefix;
}

// Exact threshold over the whole row: value-bin histogram, the bin's key
// interval, a ballot pass that writes the kept bitmap above the interval and
// lists the keys inside it, then radix select over that list (or over the
// whole row if the list would overflow).  Marks keys above T in keepmap and
// keys equal to T in tiemap; returns `need`, the number of ties to keep.
template <class G>
__device__ __forceinline__ uint32_t exact_path(const float* row, int n, int B, int lcap, const Smem& m, Scratch<G>& S) {
  const int lane = threadIdx.x & 31, warp = G::warp();
  const int words = (n + 31) >> 5;
  G::sync();                                       // the sampled path is done with the shared arrays
  uint32_t mm[4] = {0xffffffffu, 0u, 0xffffffffu, 0u};
  for (int i = G::tid(); i < n; i += G::NT) {
    const uint32_t k = key_at(row, i);
    mm[0] = min(mm[0], k);
    mm[1] = max(mm[1], k);
    if (k > kKeyNegInf && k < kKeyPosInf) {
      mm[2] = min(mm[2], k);
      mm[3] = max(mm[3], k);
    }
  }
  for (int w = G::tid(); w < words; w += G::NT) m.tiemap[w] = 0u;
  if (G::tid() == 0) S.count = 0;
  group_minmax4<G>(mm, S);
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
    for (int i = G::tid(); i < kBins; i += G::NT) S.hist[i] = 0;
    G::sync();
    for (int i = G::tid(); i < n; i += G::NT) atomicAdd(&S.hist[value_bin(key_at(row, i), scale, lo_s)], 1u);
    G::sync();
    check_hist_total<G>(S.hist, kBins, static_cast<uint32_t>(n), S.scan);
    uint32_t above;
    const int bin = find_digit<G>(S.hist, kBins, need, S, &above);
    need -= above;
    ncand = S.hist[bin];
    if (warp == 0) {
      const uint64_t k0 = first_key_in_bin(bin, scale, lo_s);
      const uint64_t k1 = bin + 1 < kBins ? first_key_in_bin(bin + 1, scale, lo_s) : (uint64_t{1} << 32);
      if (lane == 0) {
        S.bounds[0] = static_cast<uint32_t>(k0);
        S.bounds[1] = static_cast<uint32_t>(k1 - 1);
      }
    }
    G::sync();
    cmin = S.bounds[0];
    cmax = S.bounds[1];
  }
  const bool listed = ncand <= static_cast<uint32_t>(lcap);
  for (int base = warp * 32; base < n; base += G::NT) {
    const int i = base + lane;
    const bool in = i < n;
    const uint32_t k = in ? key_at(row, i) : 0u;
    const uint32_t bits = __ballot_sync(0xffffffffu, in && k > cmax);
    if (lane == 0) m.keepmap[base >> 5] = bits;
    if (listed && in && k >= cmin && k <= cmax) {
      const uint32_t pos = atomicAdd(&S.count, 1u);
      m.list_key[pos] = k;
      m.list_idx[pos] = i;
    }
  }
  G::sync();
  if (listed) {
    const int nc = static_cast<int>(S.count);
    const uint32_t T = radix_threshold<G>(
        [&](auto fn) {
          for (int j = G::tid(); j < nc; j += G::NT) fn(m.list_key[j]);
        },
        cmin, cmax, &need, S);
    for (int j = G::tid(); j < nc; j += G::NT) {
      const uint32_t k = m.list_key[j];
      const int i = m.list_idx[j];
      if (k > T) atomicOr(&m.keepmap[i >> 5], 1u << (i & 31));
      else if (k == T) atomicOr(&m.tiemap[i >> 5], 1u << (i & 31));
    }
  } else {
    const uint32_t T = radix_threshold<G>(
        [&](auto fn) {
          for (int i = G::tid(); i < n; i += G::NT) {
            const uint32_t k = key_at(row, i);
            if (k >= cmin && k <= cmax) fn(k);
          }
        },
        cmin, cmax, &need, S);
    for (int base = warp * 32; base < n; base += G::NT) {
      const int i = base + lane;
      const uint32_t k = i < n ? key_at(row, i) : 0u;
      const uint32_t mk = __ballot_sync(0xffffffffu, i < n && k > T);
      const uint32_t mt = __ballot_sync(0xffffffffu, i < n && k == T);
      if (lane == 0) {
        m.keepmap[base >> 5] = mk;
        m.tiemap[base >> 5] = mt;
      }
    }
  }
  G::sync();
  return need;
}

// Threshold among the listed keys (all in [lo_key, hi_key]): the need-th
// largest.  Value bins over [lo_key, hi_key] locate the bin that holds it; if
// that bin holds at most kSmallBin listed keys, each of them is ranked
// against the others; otherwise (crowded bin, or a range that cannot be
// binned) a radix select over the bin finishes.  *need becomes the number of
// keys equal to T to keep.
constexpr int kSmallBin = 256;

template <class G>
__device__ __forceinline__ uint32_t list_threshold(const Smem& m, int nc, uint32_t lo_key, uint32_t hi_key,
                                                   uint32_t* need, Scratch<G>& S, uint32_t* small) {
  auto all = [&](auto fn) {
    for (int j = G::tid(); j < nc; j += G::NT) fn(m.list_key[j]);
  };
  bool binned = false;
  float scale = 0.f, lo_s = 0.f;
  if (lo_key < hi_key && lo_key > kKeyNegInf && hi_key < kKeyPosInf) {
    const float lo = key_value(lo_key);
    const float width = key_value(hi_key) - lo;
    scale = static_cast<float>(kBins) / width;
    lo_s = lo * scale;
    binned = width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s);
  }
  if (!binned) return radix_threshold<G>(all, lo_key, hi_key, need, S);
  for (int i = G::tid(); i < kBins; i += G::NT) S.hist[i] = 0;
  if (G::tid() == 0) S.count = 0;
  G::sync();
  for (int j = G::tid(); j < nc; j += G::NT) atomicAdd(&S.hist[value_bin(m.list_key[j], scale, lo_s)], 1u);
  G::sync();
  check_hist_total<G>(S.hist, kBins, static_cast<uint32_t>(nc), S.scan);
  uint32_t above;
  const int bin = find_digit<G>(S.hist, kBins, *need, S, &above);
  *need -= above;
  const uint32_t inbin = S.hist[bin];
  if (inbin > static_cast<uint32_t>(kSmallBin)) {
    return radix_threshold<G>(
        [&](auto fn) {
          for (int j = G::tid(); j < nc; j += G::NT) {
            const uint32_t k = m.list_key[j];
            if (value_bin(k, scale, lo_s) == bin) fn(k);
          }
        },
        lo_key, hi_key, need, S);
  }
  for (int j = G::tid(); j < nc; j += G::NT) {
    const uint32_t k = m.list_key[j];
    if (value_bin(k, scale, lo_s) == bin) small[atomicAdd(&S.count, 1u)] = k;
  }
  G::sync();
  const int c2 = static_cast<int>(S.count);
  for (int j = G::tid(); j < c2; j += G::NT) {
    const uint32_t k = small[j];
    uint32_t gt = 0, eq = 0;
    for (int t = 0; t < c2; ++t) {
      gt += small[t] > k;
      eq += small[t] == k;
    }
    if (gt < *need && gt + eq >= *need) {
      S.bounds[0] = k;
      S.bounds[1] = *need - gt;
    }
  }
  G::sync();
  const uint32_t T = S.bounds[0];
  *need = S.bounds[1];
  G::sync();
  return T;
}

// Sampled path.  kSamples evenly spaced scores give a key L that at least
// `r` samples reach, r chosen well above the B/n share of the samples, so
// that (for any but a pathological order of the scores) between B and lcap
// keys of the row are >= L.  Two passes list exactly those keys (count with
// several loads in flight, scan, write); the B-th largest of the list is then
// the B-th largest of the row.  Returns false (having marked nothing) when
// the count falls outside [B, lcap].
template <class G>
__device__ __forceinline__ bool sampled_path(const float* row, int n, int B, int lcap, const Smem& m, Scratch<G>& S,
                                             uint32_t* need_out) {
  const int lane = threadIdx.x & 31, warp = G::warp();
  const int words = (n + 31) >> 5;
  constexpr int U = 8;
  // samples: kSamples / 8 evenly spaced chunks of 8 consecutive keys (whole
  // 32-byte sectors, so the sample costs 1/8 of a pass over the row)
  const int chunks = min((n + 7) / 8, kSamples / 8);
  const int ms = n < 8 * chunks ? n : 8 * chunks;
  const float qm = static_cast<float>(B) * static_cast<float>(ms) / static_cast<float>(n);
  const int r = static_cast<int>(ceilf(qm + 5.f * sqrtf(qm) + 20.f));
  for (int w = G::tid(); w < words; w += G::NT) {
    m.keepmap[w] = 0u;
    m.tiemap[w] = 0u;
  }
  // r >= ms: every key will be listed, whatever the samples say (rows only a
  // little longer than B), so they are not drawn
  uint32_t mm[4] = {0xffffffffu, 0u, 0xffffffffu, 0u};
  if (r < ms) {
    for (int q = G::tid(); q < chunks; q += G::NT) {
      const int i0 = n <= 8 * chunks ? 8 * q : static_cast<int>(static_cast<int64_t>(q) * (n / 8) / chunks) * 8;
      float v[8];
      if (i0 + 7 < n) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(row + i0));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(row + i0 + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = 0.f;
        for (int e = 0; i0 + e < n && e < 8; ++e) v[e] = __ldcg(row + i0 + e);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = 8 * q + e;
        if (j < ms) {
          const uint32_t k = order_key(v[e]);
          m.samples[j] = k;
          if (k > kKeyNegInf && k < kKeyPosInf) {
            mm[2] = min(mm[2], k);
            mm[3] = max(mm[3], k);
          }
        }
      }
    }
    group_minmax4<G>(mm, S);
  }
  uint32_t L = 0u;                                 // r >= ms: every key is listed
  if (r < ms) {
    if (!(mm[2] < mm[3])) return false;            // no spread among the samples
    const float lo = key_value(mm[2]);
    const float width = key_value(mm[3]) - lo;
    const float scale = static_cast<float>(kBins) / width;
    const float lo_s = lo * scale;
    if (!(width > 0.f && isfinite(width) && isfinite(scale) && scale > 0.f && isfinite(lo_s))) return false;
    for (int i = G::tid(); i < kBins; i += G::NT) S.hist[i] = 0;
    G::sync();
    for (int j = G::tid(); j < ms; j += G::NT) atomicAdd(&S.hist[value_bin(m.samples[j], scale, lo_s)], 1u);
    G::sync();
    uint32_t above;
    const int bin = find_digit<G>(S.hist, kBins, static_cast<uint32_t>(r), S, &above);
    if (warp == 0) {
      const uint64_t k0 = first_key_in_bin(bin, scale, lo_s);
      if (lane == 0) S.bounds[0] = static_cast<uint32_t>(k0);
    }
    G::sync();
    L = S.bounds[0];
  }
  // list every key >= L: U float4 loads in flight per thread, one
  // warp-aggregated reservation per warp and pass step.  Only the indices go
  // into the list here (walking the set bits of a lane's flags, with no
  // per-element work); the keys are read back from the row afterwards.
  if (G::tid() == 0) S.count = 0;
  G::sync();
  // key >= L as a float comparison: L = 0 takes every key (NaN included);
  // L at or below -inf's key takes every number; otherwise key >= L exactly
  // when score >= value(L) (-0 and +0 compare equal, NaN compares false).
  const bool take_all = L == 0u;
  const float Lv = L <= kKeyNegInf ? -INFINITY : key_value(L);
  for (int w0 = warp * 32 * 4 * U; w0 < n; w0 += G::NT * 4 * U) {
    float4 v[U];
    uint32_t flags = 0u;       // bit 4e+q: key w0 + (32e + lane)*4 + q is >= L
    if (w0 + 32 * 4 * U <= n) {                    // warp-uniform: a full step
#pragma unroll
      for (int e = 0; e < U; ++e) v[e] = __ldcg(reinterpret_cast<const float4*>(row + w0 + (e * 32 + lane) * 4));
#pragma unroll
      for (int e = 0; e < U; ++e) {
        flags |= static_cast<uint32_t>(take_all || v[e].x >= Lv) << (4 * e);
        flags |= static_cast<uint32_t>(take_all || v[e].y >= Lv) << (4 * e + 1);
        flags |= static_cast<uint32_t>(take_all || v[e].z >= Lv) << (4 * e + 2);
        flags |= static_cast<uint32_t>(take_all || v[e].w >= Lv) << (4 * e + 3);
      }
    } else {
#pragma unroll
      for (int e = 0; e < U; ++e) {
        const int i = w0 + (e * 32 + lane) * 4;
        if (i + 3 < n) v[e] = __ldcg(reinterpret_cast<const float4*>(row + i));
        else v[e] = make_float4(i < n ? __ldcg(row + i) : 0.f, i + 1 < n ? __ldcg(row + i + 1) : 0.f,
                                i + 2 < n ? __ldcg(row + i + 2) : 0.f, 0.f);
      }
#pragma unroll
      for (int e = 0; e < U; ++e) {
        const int i = w0 + (e * 32 + lane) * 4;
        const float t[4] = {v[e].x, v[e].y, v[e].z, v[e].w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          flags |= static_cast<uint32_t>(i + q < n && (take_all || t[q] >= Lv)) << (4 * e + q);
      }
    }
    const uint32_t cnt = __popc(flags);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t base = 0u;
    if (lane == 0 && total) base = atomicAdd(&S.count, total);
    uint32_t pos = __shfl_sync(0xffffffffu, base, 0) + incl - cnt;
    while (flags) {
      const int bit = __ffs(flags) - 1;
      flags &= flags - 1u;
      if (pos < static_cast<uint32_t>(lcap)) m.list_idx[pos] = w0 + ((bit >> 2) * 32 + lane) * 4 + (bit & 3);
      ++pos;
    }
  }
  G::sync();                                       // the list's indices and its count are complete
  const uint32_t c = S.count;
  // the listed keys, and the largest of them (NaN keys are 0, below every bound)
  uint32_t lmax = L;
  for (int jj = G::tid(); jj < min(static_cast<int>(c), lcap); jj += G::NT) {
    const uint32_t k = order_key(__ldcg(row + m.list_idx[jj]));
    m.list_key[jj] = k;
    lmax = max(lmax, k);
  }
  lmax = __reduce_max_sync(0xffffffffu, lmax);
  if (lane == 0) S.red[1][warp] = lmax;
  G::sync();
  uint32_t hi = 0u;
  for (int w = 0; w < G::NW; ++w) hi = max(hi, S.red[1][w]);
  const bool ok = c >= static_cast<uint32_t>(B) && c <= static_cast<uint32_t>(lcap);
  G::sync();                                       // every thread has read count and red
  if (!ok) return false;
  uint32_t need = static_cast<uint32_t>(B);
  const int nc = static_cast<int>(c);
  const uint32_t T = list_threshold<G>(m, nc, L, hi, &need, S, S.small);
  for (int j = G::tid(); j < nc; j += G::NT) {
    const uint32_t k = m.list_key[j];
    const int i = m.list_idx[j];
    if (k > T) atomicOr(&m.keepmap[i >> 5], 1u << (i & 31));
    else if (k == T) atomicOr(&m.tiemap[i >> 5], 1u << (i & 31));
  }
  G::sync();
  *need_out = need;
  return true;
}

// Select one row of n > B scores: writes the B kept indices, ascending, to kept.
template <class G>
__device__ __forceinline__ void select_row(const float* row, int n, int B, int lcap, const Smem& m, Scratch<G>& S,
                                           int32_t* kept) {
  uint32_t need;
  if (!sampled_path<G>(row, n, B, lcap, m, S, &need)) need = exact_path<G>(row, n, B, lcap, m, S);

  // ties: keep the `need` lowest indices equal to T; then write out in index order
  const int words = (n + 31) >> 5;
  const int per = (words + G::NT - 1) / G::NT;        // words per thread, contiguous
  const int w0 = min(words, G::tid() * per);
  const int w1 = min(words, w0 + per);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(m.tiemap[w]);
  uint32_t total;
  uint32_t before = group_exclusive_sum<G>(cnt, S.scan, &total);
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
  G::sync();
  cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(m.keepmap[w]);
  uint32_t slot = group_exclusive_sum<G>(cnt, S.scan, &total);
  if (G::tid() == 0) TRI_CHECK(total == static_cast<uint32_t>(B));     // exactly B kept
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = m.keepmap[w];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      kept[slot++] = w * 32 + bit;
      bits &= bits - 1u;
    }
  }
  G::sync();                                       // the shared arrays may be reused next
}

template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) select_kernel(const __grid_constant__ Geom g, const Args a) {
  using G = Group<NT, 0, 0>;
  extern __shared__ uint4 select_dyn[];
  __shared__ Scratch<G> S;
  const int u = blockIdx.x;
  const int b = u % g.batch;
  const int n = g.len[b];
  const int B = a.B;
  const float* row = a.scores + static_cast<int64_t>(u) * g.score_stride;
  int32_t* __restrict__ kept = a.kept + static_cast<int64_t>(u) * B;

  if (threadIdx.x == 0) a.kept_count[u] = min(n, B);
  if (n <= B) {
    for (int i = threadIdx.x; i < n; i += NT) kept[i] = i;
    return;
  }
  const Smem m = carve(reinterpret_cast<uint32_t*>(select_dyn), a.cap, a.lcap);
  select_row<G>(row, n, B, a.lcap, m, S, kept);
}

// Capacity of the key list for budget B on rows of at most `cap` keys.
inline int list_capacity(int B, int cap) {
  const int64_t want = int64_t{B} + B / 2 + 2048;
  return static_cast<int>(want < cap ? want : cap);
}

// Dynamic shared memory of one row's selection.
inline size_t smem_bytes(int cap, int lcap) {
  const int64_t wcap = (int64_t{cap} + 31) / 32;
  const int64_t keys = lcap > kSamples ? lcap : kSamples;
  return static_cast<size_t>(keys + int64_t{lcap} + 2 * wcap) * 4;
}

}  // namespace select
}  // namespace tri
