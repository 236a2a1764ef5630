// One kernel for the whole step of a cache with few units (score, keep the
// top B, compact K and V), for CONTIG and RAGGED caches compacted out of place.
// The step is the one of the page "The future-offset average in TriAttention
// can be precomputed": the folded score of its section "The averaging step -
// the one we improve" (one dot product per key with the folded weights), then
// the opening section's keep-the-highest-within-budget and evict-the-rest.
//
// With few units, the three-kernel path is latency-bound: selection runs one
// CTA per unit, so a handful of SMs work while the rest idle.  Here each unit
// gets a thread-block cluster of kCluster CTAs:
//  1. score: every CTA streams its slice of the unit's keys (at most
//     kMaxSlice keys) through a ring of bulk copies, exactly as the
//     standalone scorer does (same lanes, same summation order, so the scores
//     are bit-identical), and keeps the order keys of its scores in its own
//     shared memory (the fp32 scores also go to the workspace);
//  2. select: a radix select over the cluster finds the order key T of the
//     B-th largest score and how many keys equal to T stay: per digit pass
//     (11, 11, 10 bits) each CTA histograms its slice, CTA r sums bins
//     [r S, r S + S) over the cluster through distributed shared memory, and
//     every CTA reads the segment totals and the one segment that holds the
//     B-th key (loads and stores of peer shared memory only);
//  3. emit: keys above T are kept, and the ties with the lowest indices: the
//     slices are in index order, so a CTA's share of the ties and its output
//     offset come from the counts of the CTAs before it; each CTA writes its
//     kept indices in ascending order and copies their K and V rows.
// The order (score descending, index ascending, NaN lowest, -0 = +0) is the
// one of select.cuh, so the kept set equals the three-kernel path's.
//
// Every CTA reaches every cluster barrier (no early exit: a timed-out wait in
// the score phase only sets the status word), and the last barrier keeps each
// CTA's shared memory alive until its peers are done reading it.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "score.cuh"
#include "select.cuh"

namespace tri {
namespace fused {

namespace cg = cooperative_groups;

constexpr int kThreads = score::kThreads;           // 8 consumer warps + 1 producer warp during scoring
constexpr int kStages = 2;                          // two CTAs fit an SM, so a wave holds every cluster
constexpr int kMaxSlice = 4096;                     // keys per CTA
constexpr int kMaxRow = 8192;                       // longest row the host sends here
constexpr int kBins = 2048;
constexpr size_t kStageBytes = score::kTileBytes;
constexpr size_t kKeysOffset = kStages * kStageBytes;                      // uint32 [kMaxSlice]
constexpr size_t kHistOffset = kKeysOffset + kMaxSlice * 4;                // uint32 [kBins]
constexpr size_t kSegOffset = kHistOffset + kBins * 4;                     // uint32 [kBins + 256]: segment, partials
constexpr size_t kMiscOffset = kSegOffset + (kBins + 256) * 4;             // exchange words, scan scratch
constexpr size_t kBarOffset = kMiscOffset + 256;
constexpr size_t kSmemBytes = kBarOffset + 2 * kStages * sizeof(uint64_t);

// Words of the misc area (uint32 index).
enum Misc : int {
  kSegTotal = 0,    // this CTA's segment total (per pass)
  kGtCount = 1,     // keys of the slice above T
  kEqCount = 2,     // keys of the slice equal to T
  kAbort = 3,
  kPrefix = 4,      // broadcast of the pass result: prefix, mask, remaining rank
  kMask = 5,
  kRank = 6,
  kScan = 16,       // block scan scratch (kThreads / 32 words)
};

struct Args {
  const float* w;        // folded weights [L*H][128]
  float* scores;         // [units][stride]
  int32_t* kept;         // [units][B]
  int32_t* kept_count;   // [units]
  uint16_t* k_out;       // [units][B][128]
  uint16_t* v_out;
  int B;
  int slice;             // keys per CTA (multiple of 128, <= kMaxSlice)
};

template <int C>
__global__ void __launch_bounds__(kThreads, 2) fused_kernel(const __grid_constant__ Geom g, const Args a) {
  static_assert(C >= 8 && C <= 32 && kBins / C % 32 == 0 && kBins / C / 32 <= 8, "cluster size");
  extern __shared__ __align__(1024) unsigned char smem[];
  uint32_t* sk = reinterpret_cast<uint32_t*>(smem + kKeysOffset);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kHistOffset);
  uint32_t* seg = reinterpret_cast<uint32_t*>(smem + kSegOffset);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kMiscOffset);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the unit of this cluster and the CTA's slice of it
  const int u = blockIdx.x / C;
  const int b = u % g.batch, lh = u / g.batch;
  const int l = lh / g.H, h = lh - l * g.H;
  const int n = g.len[b];
  const int s0 = min(n, rank * a.slice);
  const int n_loc = min(n, s0 + a.slice) - s0;
  float* srow = a.scores + static_cast<int64_t>(u) * g.score_stride;

  for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0u;
  if (threadIdx.x == 0) {
    misc[kAbort] = 0u;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], score::kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ---------------------------------------------------------------- 1. score
  const int ntiles = (n_loc + score::kTileRows - 1) / score::kTileRows;
  if (warp == score::kConsumerWarps) {
    if (lane == 0) {
      const uint64_t policy = policy_evict_first();
      bool ok = true;
      int k = 0;
      for (; k < ntiles; ++k) {
        const int s = k % kStages, nn = k / kStages;
        if (nn > 0 && !mbar_wait_bounded(&empty[s], (nn - 1) & 1)) {
          misc[kAbort] = 1u;
          break;
        }
        const int i0 = s0 + k * score::kTileRows;
        const uint32_t bytes = static_cast<uint32_t>(min(score::kTileRows, s0 + n_loc - i0)) * kRowBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(smem + static_cast<size_t>(s) * kStageBytes, g.k + row_elem(g, l, h, b, i0, &ok), bytes, &full[s],
                 policy);
      }
      for (int s = 0; s < kStages && s < k; ++s) mbar_wait_bounded(&full[s], ((k - 1 - s) / kStages) & 1);
    }
  } else {
    // 4 lanes per key, the odd key of a quarter-warp reading its chunks rotated
    const int c = lane & 3, r8 = lane >> 2, p = r8 & 1;
    const int row0 = warp * score::kRowsPerWarpPass + r8;
    float wv[32];
    score::load_w(a.w, lh, c, p, wv);
    for (int k = 0; k < ntiles; ++k) {
      const int s = k % kStages, nn = k / kStages;
      if (!mbar_wait_bounded(&full[s], nn & 1)) {
        misc[kAbort] = 1u;
        break;
      }
      const int rows = min(score::kTileRows, n_loc - k * score::kTileRows);
      const unsigned char* buf = smem + static_cast<size_t>(s) * kStageBytes;
#pragma unroll
      for (int it = 0; it < score::kIters; ++it) {
        const int r = it * score::kGroup + row0;
        uint4 x[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          x[q] = *reinterpret_cast<const uint4*>(buf + r * kRowBytes + (4 * (q ^ p) + c) * 16);
        float d[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) d[q] = score::dot8(x[q], wv + 8 * q, 0.f);
        float v = (d[0] + d[1]) + (d[2] + d[3]);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (c == 0 && r < rows) {
          const int i = k * score::kTileRows + r;
          sk[i] = select::order_key(v);
          srow[s0 + i] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  __syncthreads();   // the slice's order keys are complete; the stages are free

  // ---------------------------------------------------------------- 2. select
  const int M = min(a.B, n);
  uint32_t T = 0u, need = 0u;
  if (n > a.B) {
    uint32_t prefix = 0u, mask = 0u, R = static_cast<uint32_t>(a.B);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0;
      const int nb = pass == 2 ? 1024 : 2048;
      const uint32_t dmask = static_cast<uint32_t>(nb - 1);
      // leading digits of fp32 scores crowd into a few bins: one atomic per
      // group of lanes holding the same bin
      for (int i0 = warp * 32; i0 < n_loc; i0 += kThreads) {
        const int i = i0 + lane;
        const uint32_t key = i < n_loc ? sk[i] : 0u;
        const bool in = i < n_loc && (key & mask) == prefix;
        const uint32_t bin = in ? (key >> shift) & dmask : 0xffffffffu;
        const uint32_t same = __match_any_sync(0xffffffffu, bin);
        if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(same)));
      }
      cluster.sync();                                   // every histogram complete
      const int S = nb / C;                             // bins per segment (64 .. 256)
      // 256 threads: G = 256 / S threads per bin, each summing C / G ranks (independent loads)
      const int G = 256 / S;
      uint32_t part = 0u;
      if (threadIdx.x < 256) {
        const int t = threadIdx.x % S, grp = threadIdx.x / S;
        const int nq = C / G;                           // C and G are powers of two, G <= C
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          v[j] = j < nq ? cluster.map_shared_rank(hist, grp * nq + j)[rank * S + t] : 0u;
#pragma unroll
        for (int j = 0; j < 16; ++j) part += v[j];
        seg[kBins + threadIdx.x] = part;                 // partial sums, combined below
      }
      __syncthreads();
      uint32_t mine = 0u;
      if (threadIdx.x < S) {
        for (int grp = 0; grp < G; ++grp) mine += seg[kBins + grp * S + threadIdx.x];
        seg[threadIdx.x] = mine;
      }
      uint32_t total;
      block_exclusive_sum<kThreads>(mine, misc + kScan, &total);
      if (threadIdx.x == 0) misc[kSegTotal] = total;
      cluster.sync();                                   // every segment and total complete
      for (int i = threadIdx.x; i < nb; i += kThreads) hist[i] = 0u;
      if (warp == 0) {
        // segment holding the R-th largest key: suffix sums of the totals, from the top
        const uint32_t tot = lane < C ? cluster.map_shared_rank(misc, lane)[kSegTotal] : 0u;
        uint32_t suf = tot;                             // totals of segments >= lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 32) suf += y;
        }
        const uint32_t above = suf - tot;               // keys in segments above lane
        const int sstar = 31 - __clz(__ballot_sync(0xffffffffu, lane < C && above < R && R <= suf));
        const uint32_t R1 = R - __shfl_sync(0xffffffffu, above, sstar);
        // the bin inside that segment: S / 32 bins per lane, highest bins in lane 31
        const uint32_t* sg = cluster.map_shared_rank(seg, sstar);
        const int per = S / 32;                         // S is a multiple of 32, per <= 8
        uint32_t cnt[8];
        uint32_t lsum = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          cnt[j] = j < per ? sg[lane * per + j] : 0u;
          lsum += cnt[j];
        }
        uint32_t lsuf = lsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, lsuf, o);
          if (lane + o < 32) lsuf += y;
        }
        const uint32_t labove = lsuf - lsum;
        const int lstar = 31 - __clz(__ballot_sync(0xffffffffu, labove < R1 && R1 <= lsuf));
        if (lane == lstar) {
          uint32_t acc = labove;
          int bin = -1;
#pragma unroll
          for (int j = 7; j >= 0; --j) {
            if (bin < 0 && j < per) {
              if (acc + cnt[j] >= R1) bin = lane * per + j;
              else acc += cnt[j];
            }
          }
          const uint32_t digit = static_cast<uint32_t>(sstar * S + bin);
          misc[kPrefix] = prefix | (digit << shift);
          misc[kMask] = mask | (dmask << shift);
          misc[kRank] = R1 - acc;
        }
      }
      __syncthreads();
      prefix = misc[kPrefix];
      mask = misc[kMask];
      R = misc[kRank];
      __syncthreads();
    }
    T = prefix;
    need = R;                                           // keys equal to T that stay
  }

  // ---------------------------------------------------------------- 3. emit
  uint32_t gt = 0u, eq = 0u;
  for (int i = threadIdx.x; i < n_loc; i += kThreads) {
    const uint32_t key = sk[i];
    gt += n > a.B ? (key > T) : 1u;                     // n <= B: every key stays
    eq += n > a.B ? (key == T) : 0u;
  }
  uint32_t gt_all, eq_all;
  block_exclusive_sum<kThreads>(gt, misc + kScan, &gt_all);
  block_exclusive_sum<kThreads>(eq, misc + kScan, &eq_all);
  if (threadIdx.x == 0) {
    misc[kGtCount] = gt_all;
    misc[kEqCount] = eq_all;
  }
  cluster.sync();                                       // every CTA's counts published
  // ties before this slice, and kept keys before this slice: warp 0 reads every
  // CTA's counts at once, prefix sums over the lanes
  if (warp == 0) {
    uint32_t eq_q = 0u, gt_q = 0u;
    if (lane < C) {
      const uint32_t* m = cluster.map_shared_rank(misc, lane);
      eq_q = m[kEqCount];
      gt_q = m[kGtCount];
    }
    uint32_t eq_incl = eq_q;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, eq_incl, o);
      if (lane >= o) eq_incl += y;
    }
    const uint32_t eq_excl = eq_incl - eq_q;             // ties in slices before lane
    const uint32_t take = need > eq_excl ? min(eq_q, need - eq_excl) : 0u;
    uint32_t kept_incl = gt_q + take;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, kept_incl, o);
      if (lane >= o) kept_incl += y;
    }
    if (lane == rank) {
      misc[kPrefix] = kept_incl - (gt_q + take);         // output offset of this slice
      misc[kMask] = take;                                // ties this slice keeps
    }
  }
  __syncthreads();
  const uint32_t out_off = misc[kPrefix];
  const uint32_t keep_eq = misc[kMask];
  // kept indices in ascending order; their slice offsets go to the (free)
  // stage memory.  Each warp takes a contiguous run of the slice, ranks by
  // ballot and popcount, and the runs are ordered by two rounds of per-warp
  // totals.
  int32_t* list = reinterpret_cast<int32_t*>(smem);
  int32_t* kept_row = a.kept + static_cast<int64_t>(u) * a.B;
  uint32_t* wtot = misc + kScan;                         // per-warp totals
  constexpr int NW = kThreads / 32;
  const int run = (n_loc + NW * 32 - 1) / (NW * 32) * 32;
  const int w0 = min(n_loc, warp * run), w1 = min(n_loc, w0 + run);
  const uint32_t lt = (1u << lane) - 1u;
  const bool sel = n > a.B;
  uint32_t e_cnt = 0u;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    e_cnt += __popc(__ballot_sync(0xffffffffu, i < w1 && sel && sk[i] == T));
  }
  if (lane == 0) wtot[warp] = e_cnt;
  __syncthreads();
  uint32_t e_prefix = 0u;                                // ties before this warp's run
  for (int q = 0; q < warp; ++q) e_prefix += wtot[q];
  __syncthreads();                                       // (wtot is reused below)
  uint32_t e_run = e_prefix, k_cnt = 0u;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < w1 ? sk[i] : 0u;
    const uint32_t em = __ballot_sync(0xffffffffu, i < w1 && sel && key == T);
    const bool keep = i < w1 && (!sel || key > T || ((em >> lane & 1u) && e_run + __popc(em & lt) < keep_eq));
    k_cnt += __popc(__ballot_sync(0xffffffffu, keep));
    e_run += __popc(em);
  }
  if (lane == 0) wtot[warp] = k_cnt;
  __syncthreads();
  uint32_t k_run = 0u, kept_base = 0u;                   // kept before this run; kept in the slice
  for (int q = 0; q < NW; ++q) {
    kept_base += wtot[q];
    if (q < warp) k_run += wtot[q];
  }
  e_run = e_prefix;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < w1 ? sk[i] : 0u;
    const uint32_t em = __ballot_sync(0xffffffffu, i < w1 && sel && key == T);
    const bool keep = i < w1 && (!sel || key > T || ((em >> lane & 1u) && e_run + __popc(em & lt) < keep_eq));
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    const uint32_t pos = k_run + __popc(km & lt);
    if (keep && out_off + pos < static_cast<uint32_t>(a.B)) {   // (only a timed-out wait can break the bound)
      kept_row[out_off + pos] = s0 + i;
      list[pos] = i;
    }
    k_run += __popc(km);
    e_run += __popc(em);
  }
  __syncthreads();
  // copy the kept rows: 16 threads per row, 16 bytes each, K then V
  const int nk = static_cast<int>(min(kept_base, out_off < static_cast<uint32_t>(a.B) ? a.B - out_off : 0u));
  const int64_t out0 = static_cast<int64_t>(u) * a.B + out_off;
  const int sub = threadIdx.x & 15;
  constexpr int kRowsPerPass = kThreads / 16;
  for (int j0 = threadIdx.x >> 4; j0 < nk; j0 += 4 * kRowsPerPass) {
    uint4 kv[4], vv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + q * kRowsPerPass;
      if (j < nk) {
        bool ok = true;
        const int64_t src = row_elem(g, l, h, b, s0 + list[j], &ok);
        kv[q] = *reinterpret_cast<const uint4*>(g.k + src + sub * 8);
        vv[q] = *reinterpret_cast<const uint4*>(g.v + src + sub * 8);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + q * kRowsPerPass;
      if (j < nk) {
        *reinterpret_cast<uint4*>(a.k_out + (out0 + j) * kD + sub * 8) = kv[q];
        *reinterpret_cast<uint4*>(a.v_out + (out0 + j) * kD + sub * 8) = vv[q];
      }
    }
  }
  if (rank == 0 && threadIdx.x == 0) a.kept_count[u] = M;
  // the last slice's kept keys end the unit's list at exactly M
  if (rank == C - 1 && threadIdx.x == 0 && !misc[kAbort]) TRI_CHECK(out_off + kept_base == static_cast<uint32_t>(M));
  if (threadIdx.x == 0 && misc[kAbort]) flag(TRI_DEVFLAG_TIMEOUT);
  cluster.sync();                                       // peers are done with this CTA's shared memory
}

}  // namespace fused
}  // namespace tri
