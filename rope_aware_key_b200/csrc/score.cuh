// Scoring: scores[u][i] = sum_j w[l*H + h][j] * float(K_u[i][j]).
//
// This is the folded score of the page "The future-offset average in
// TriAttention can be precomputed" (section "The averaging step - the one we
// improve"): after the fold, one evaluation per key instead of one per
// offset.  128 FMAs per 256-byte key, so the kernel is bound by HBM: it is a
// stream of the key cache through shared memory.
//
// Design (persistent, TRI_SCORE_CTAS_PER_SM CTAs per SM):
//  * a producer warp decodes the CTA's next kPreTiles tiles at once, one
//    lane per tile -- up to 128 consecutive keys of one unit (CONTIG,
//    RAGGED) or consecutive pages of all heads (PAGED), whose page ids come
//    from the block table in global memory, so the lookups of a batch
//    overlap -- then one lane writes each tile's metadata next to its stage
//    and issues its 1-D bulk copies (cp.async.bulk, no multicast, L2
//    evict-first) into a ring of TRI_SCORE_STAGES 32 KB shared-memory stages
//    guarded by full/empty mbarriers;
//  * 8 consumer warps read a stage with 16-byte shared loads, four lanes per
//    key (32 bf16 each).  The two keys of a quarter-warp read opposite halves
//    of the 128-byte bank window at every load (the odd key's chunk order is
//    rotated), so the loads are conflict-free; each lane keeps its 32
//    weights in registers in its own rotated order.  Two shuffles reduce a
//    key;
//  * every wait is bounded (about 2 s) and reported through the status word.
#pragma once

#include "common.cuh"

#ifndef TRI_SCORE_STAGES
#define TRI_SCORE_STAGES 3
#endif
#ifndef TRI_SCORE_CTAS_PER_SM
#define TRI_SCORE_CTAS_PER_SM 2
#endif

namespace tri {
namespace score {

constexpr int kTileRows = 128;
constexpr int kTileBytes = kTileRows * kRowBytes;   // 32 KB
constexpr int kStages = TRI_SCORE_STAGES;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kRowsPerWarpPass = 8;                  // 4 lanes per key
constexpr int kGroup = kRowsPerWarpPass * kConsumerWarps;   // rows per pass of all consumers
constexpr int kIters = kTileRows / kGroup;

// Decoded tile, written by the producer next to its stage.
struct TileInfo {
  int rows;          // rows held in the stage (0: nothing to do)
  int paged;         // rows interleave heads (PAGED)
  int lh;            // layer*H + head of row 0 (CONTIG / RAGGED), layer*H (PAGED)
  int tvalid;        // PAGED: tokens of the tile inside the sequence
  int page0;         // PAGED: the tile's first page (index in the sequence's block table)
  int pages;         // PAGED: pages in the tile (their rows follow one another in the stage)
  uint32_t page_ok;  // PAGED: bit p set when page p of the tile has a valid id (and was copied)
  int b;             // sequence
  int i0;            // index in the sequence of the tile's first key
  int tq;            // distance scorers: the query position of sequence b
  float* out;        // score of row 0 (CONTIG / RAGGED) or of head 0, token 0 (PAGED)
  int64_t head_step; // PAGED: floats between the score rows of consecutive heads
};

// Tiles decoded ahead by the producer warp (one lane each), with the first
// kPrePages page ids of a PAGED tile.
constexpr int kPreTiles = 16;
constexpr int kPrePages = 8;
struct PreTile {
  TileInfo T;
  int64_t src;
  int32_t blk[kPrePages];
  int ok;
};

constexpr size_t kBarOffset = static_cast<size_t>(kStages) * kTileBytes;
constexpr size_t kInfoOffset = kBarOffset + 2 * kStages * sizeof(uint64_t);
constexpr size_t kPreOffset = (kInfoOffset + kStages * sizeof(TileInfo) + 15) & ~size_t{15};
constexpr size_t kSmemBytes = kPreOffset + kPreTiles * sizeof(PreTile);

// Tiles are numbered layer-major: CONTIG / RAGGED per (layer, head) then
// sequence then 128-key chunk; PAGED per layer then sequence then group of
// pages_per_tile consecutive pages (as many as fill 128 rows).  For PAGED,
// *src is unused: the producer copies each page of the tile on its own, and
// the first kPrePages page ids go to blk when it is given.
__device__ __forceinline__ void decode(const Geom& g, int t, float* scores, TileInfo* T, int64_t* src,
                                       bool* ok, int32_t* blk_out = nullptr) {
  const int per = g.tile_prefix[g.batch];
  const int outer = t / per;
  const int r = t - outer * per;
  const int b = find_seq(g.tile_prefix, g.batch, r);
  const int j = r - g.tile_prefix[b];
  *ok = true;
  T->b = b;
  if (g.layout == TRI_LAYOUT_PAGED) {
    const int l = outer;
    const int P = g.pages_per_tile;
    const int i0 = j * P * g.block_size;
    const int seq_pages = (g.len[b] + g.block_size - 1) / g.block_size;
    T->i0 = i0;
    T->page0 = j * P;
    T->pages = min(P, seq_pages - j * P);
    T->rows = T->pages * g.block_size * g.H;
    T->paged = 1;
    T->lh = l * g.H;
    T->tvalid = min(P * g.block_size, g.len[b] - i0);
    T->head_step = static_cast<int64_t>(g.batch) * g.score_stride;
    T->out = scores + (static_cast<int64_t>(l) * g.H * g.batch + b) * g.score_stride + i0;
    T->page_ok = 0u;
    for (int p = 0; p < T->pages; ++p) {
      const int blk = g.block_table[static_cast<int64_t>(b) * g.max_blocks + j * P + p];
      if (static_cast<unsigned>(blk) < static_cast<unsigned>(g.num_blocks)) T->page_ok |= 1u << p;
      else *ok = false;
      if (blk_out && p < kPrePages) blk_out[p] = blk;
    }
    *src = 0;
  } else {
    const int l = outer / g.H;
    const int h = outer - l * g.H;
    const int i0 = j * kTileRows;
    T->i0 = i0;
    T->rows = min(kTileRows, g.len[b] - i0);
    T->paged = 0;
    T->page0 = 0;
    T->pages = 0;
    T->page_ok = 0u;
    T->lh = outer;
    T->tvalid = T->rows;
    T->head_step = 0;
    T->out = scores + (static_cast<int64_t>(outer) * g.batch + b) * g.score_stride + i0;
    *src = row_elem(g, l, h, b, i0, ok);
  }
}

// Dot product of 8 bf16 (packed in x, element order) with 8 fp32 weights.
__device__ __forceinline__ float dot8(const uint4 x, const float* w, float a) {
  a = fmaf(__uint_as_float(x.x << 16), w[0], a);
  a = fmaf(__uint_as_float(x.x & 0xffff0000u), w[1], a);
  a = fmaf(__uint_as_float(x.y << 16), w[2], a);
  a = fmaf(__uint_as_float(x.y & 0xffff0000u), w[3], a);
  a = fmaf(__uint_as_float(x.z << 16), w[4], a);
  a = fmaf(__uint_as_float(x.z & 0xffff0000u), w[5], a);
  a = fmaf(__uint_as_float(x.w << 16), w[6], a);
  a = fmaf(__uint_as_float(x.w & 0xffff0000u), w[7], a);
  return a;
}

// The lane's 32 weights: chunk (4*(k ^ p) + c) of the head's 16 chunks of 8,
// for k = 0..3 (the order in which the lane reads a key).
__device__ __forceinline__ void load_w(const float* __restrict__ w, int lh, int c, int p, float (&wv)[32]) {
  const float4* base = reinterpret_cast<const float4*>(w + static_cast<int64_t>(lh) * kD);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int ch = 4 * (k ^ p) + c;
    const float4 a = __ldg(base + 2 * ch), b = __ldg(base + 2 * ch + 1);
    wv[8 * k + 0] = a.x; wv[8 * k + 1] = a.y; wv[8 * k + 2] = a.z; wv[8 * k + 3] = a.w;
    wv[8 * k + 4] = b.x; wv[8 * k + 5] = b.y; wv[8 * k + 6] = b.z; wv[8 * k + 7] = b.w;
  }
}

// Nothing besides the keys travels with a tile.
struct NoSideCopy {
  __device__ __forceinline__ void annotate(TileInfo&) const {}
  __device__ __forceinline__ uint32_t bytes(const TileInfo&) const { return 0; }
  __device__ __forceinline__ void issue(const TileInfo&, int, uint64_t*, uint64_t) const {}
};

// The producer warp (all 32 lanes call this).  The tiles a CTA takes are
// t_begin, t_begin + t_step, ... < t_end.  Per batch of kPreTiles of them,
// lane j decodes the j-th (page lookups included) into shared memory; then
// lane 0, in order, waits for each tile's stage to be free, writes the
// tile's metadata next to the stage and issues its bulk copy (plus the side
// copies of `side`, on the same barrier).  Before returning, lane 0 waits
// (bounded) for the last copy into every stage, so that no copy is in flight
// into the shared memory of an exiting CTA.
template <class Side = NoSideCopy>
__device__ __forceinline__ void produce(const Geom& g, float* scores, unsigned char* smem, uint64_t* full,
                                        uint64_t* empty, TileInfo* info, int t_begin, int t_end, int t_step,
                                        const Side& side = Side()) {
  const int lane = threadIdx.x & 31;
  PreTile* pre = reinterpret_cast<PreTile*>(smem + kPreOffset);
  const uint64_t policy = policy_evict_first();
  int k = 0;                                     // tiles issued (lane 0's count, shared after each batch)
  bool stop = false;
  for (int64_t t0 = t_begin; t0 < t_end && !stop; t0 += int64_t{kPreTiles} * t_step) {
    if (lane < kPreTiles) {
      const int64_t t = t0 + int64_t{lane} * t_step;
      if (t < t_end) {
        PreTile& P = pre[lane];
        bool ok;
        decode(g, static_cast<int>(t), scores, &P.T, &P.src, &ok, P.blk);
        if (!ok) flag(TRI_DEVFLAG_BAD_PAGE);       // the bad pages are skipped, the others scored
        side.annotate(P.T);
      }
    }
    __syncwarp();
    if (lane == 0) {
      for (int j = 0; j < kPreTiles; ++j) {
        const int64_t t = t0 + int64_t{j} * t_step;
        if (t >= t_end) break;
        const int s = k % kStages, n = k / kStages;
#ifdef TRI_TEST_HOOKS
        if (t == g.test_skip_tile) {               // test builds: no copy and no arrival for this tile
          ++k;
          continue;
        }
#endif
        if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) {
          stop = true;
          break;
        }
        const PreTile& P = pre[j];
        const TileInfo T = P.T;
        info[s] = T;
        if (T.rows > 0) {
          unsigned char* dst = smem + static_cast<size_t>(s) * kTileBytes;
          if (!T.paged) {
            const uint32_t bytes = static_cast<uint32_t>(T.rows) * kRowBytes;
            mbar_arrive_expect_tx(&full[s], bytes + side.bytes(T));
            bulk_g2s(dst, g.k + P.src, bytes, &full[s], policy);
          } else {
            const uint32_t page_bytes = static_cast<uint32_t>(g.block_size * g.H) * kRowBytes;
            mbar_arrive_expect_tx(&full[s], page_bytes * __popc(T.page_ok) + side.bytes(T));
            const int l = T.lh / g.H;
            for (int p = 0; p < T.pages; ++p) {
              if (!((T.page_ok >> p) & 1u)) continue;
              const int blk = p < kPrePages
                  ? P.blk[p]
                  : g.block_table[static_cast<int64_t>(T.b) * g.max_blocks + T.page0 + p];
              bulk_g2s(dst + static_cast<size_t>(p) * page_bytes,
                       g.k + l * g.sL + static_cast<int64_t>(blk) * g.sB, page_bytes, &full[s], policy);
            }
          }
          side.issue(T, s, &full[s], policy);
        } else {
          mbar_arrive(&full[s]);
        }
        ++k;
      }
    }
    stop = __shfl_sync(0xffffffffu, stop, 0);
    __syncwarp();                                  // the batch's slots may be rewritten
  }
  if (lane == 0) {
    for (int s = 0; s < kStages && s < k; ++s) {
      const int last = (k - 1 - s) / kStages;      // issues on stage s: s, s+S, ... < k
      mbar_wait_bounded(&full[s], last & 1);
    }
  }
}

// Barrier set-up shared by the score kernels.
__device__ __forceinline__ void init_ring(uint64_t* full, uint64_t* empty) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, TRI_SCORE_CTAS_PER_SM)
score_kernel(const __grid_constant__ Geom g, const float* __restrict__ w, float* __restrict__ scores,
             int ntiles) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + kInfoOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  init_ring(full, empty);

  if (warp == kConsumerWarps) {
    produce(g, scores, smem, full, empty, info, blockIdx.x, ntiles, gridDim.x);
    return;
  }

  // ---------------- consumers: 4 lanes per key
  const int c = lane & 3;                 // which 4 of the row's 16 chunks
  const int r8 = lane >> 2;               // key within the warp's group of 8
  const int p = r8 & 1;                   // chunk-order rotation of odd keys
  const int row0 = warp * kRowsPerWarpPass + r8;
  // PAGED rows interleave heads: row r is head r % H, and every row this
  // lane reads has the same r % H (kGroup and the warp offset are multiples
  // of 8, H | 8).  The lane's head, and for each pass the token of its row
  // and that token's page within the tile, are the same in every tile.
  int hp = 0, tok_it[kIters], page_it[kIters];
  int64_t hoff = 0;
  if (g.layout == TRI_LAYOUT_PAGED) {
    hp = row0 % g.H;
    hoff = hp * (static_cast<int64_t>(g.batch) * g.score_stride);
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      tok_it[it] = (it * kGroup + row0) / g.H;
      page_it[it] = tok_it[it] / g.block_size;
    }
  }
  float wv[32];
  int cur_lh = -1;
  int k = 0;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
    const int s = k % kStages, n = k / kStages;
    if (!mbar_wait_bounded(&full[s], n & 1)) break;
    const TileInfo T = info[s];
    if (T.rows > 0) {
      const int h = T.paged ? hp : 0;
      const int lh = T.lh + h;
      if (lh != cur_lh) {
        load_w(w, lh, c, p, wv);
        cur_lh = lh;
      }
      const unsigned char* buf = smem + static_cast<size_t>(s) * kTileBytes;
      const int iters = (T.rows + kGroup - 1) / kGroup;
      uint4 x[kIters][4];
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        if (it < iters) {
          const unsigned char* rowp = buf + (it * kGroup + row0) * kRowBytes;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            x[it][q] = *reinterpret_cast<const uint4*>(rowp + (4 * (q ^ p) + c) * 16);
        }
      }
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        if (it < iters) {   // warp-uniform
          // (d0 + d1) + (d2 + d3): the odd keys' rotation swaps d0/d1 and
          // d2/d3, and fp32 addition commutes, so every key is summed in the
          // same order whatever its position
          float d[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) d[q] = dot8(x[it][q], wv + 8 * q, 0.f);
          float a = (d[0] + d[1]) + (d[2] + d[3]);
          a += __shfl_xor_sync(0xffffffffu, a, 1);
          a += __shfl_xor_sync(0xffffffffu, a, 2);
          const int r = it * kGroup + row0;
          if (c == 0 && r < T.rows) {
            if (T.paged) {
              const int tok = tok_it[it];
              if (tok < T.tvalid && ((T.page_ok >> page_it[it]) & 1u)) T.out[hoff + tok] = a;
            } else {
              T.out[r] = a;
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace score
}  // namespace tri
