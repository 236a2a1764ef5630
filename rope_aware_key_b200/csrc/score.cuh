// Scoring: scores[u][i] = sum_j w[l*H + h][j] * float(K_u[i][j]).
//
// This is the folded score of the page "The future-offset average in
// TriAttention can be precomputed" (section "The averaging step - the one we
// improve"): after the fold, one evaluation per key instead of one per
// offset.  128 FMAs per 256-byte key, so the kernel is bound by HBM: it is a
// stream of the key cache through shared memory.
//
// Design (one persistent CTA per SM):
//  * a producer thread issues 1-D bulk copies (cp.async.bulk, no multicast)
//    of whole tiles -- up to 128 consecutive keys of one unit (CONTIG,
//    RAGGED) or one page of all heads (PAGED) -- into a ring of
//    TRI_SCORE_STAGES 32 KB shared-memory stages, each guarded by a
//    full/empty mbarrier pair; keys are fetched with an L2 evict-first hint;
//  * 8 consumer warps read the stage with 16-byte shared loads, a half-warp
//    per key (16 lanes x 8 bf16), multiply with the unit's weight slice held
//    in registers and reduce across the half-warp with shuffles;
//  * every wait is bounded (about 2 s) and reported through the status word.
#pragma once

#include "common.cuh"

#ifndef TRI_SCORE_STAGES
#define TRI_SCORE_STAGES 4
#endif

namespace tri {
namespace score {

constexpr int kTileRows = 128;
constexpr int kTileBytes = kTileRows * kRowBytes;  // 32 KB
constexpr int kStages = TRI_SCORE_STAGES;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kIters = kTileRows / (2 * kConsumerWarps);   // rows per half-warp per tile
constexpr size_t kSmemBytes = static_cast<size_t>(kStages) * kTileBytes + 2 * kStages * sizeof(uint64_t);

struct Tile {
  int l, h, b;     // h is meaningful for CONTIG / RAGGED only
  int i0;          // first key index of the tile
  int rows;        // rows held in the stage
  int tvalid;      // PAGED: tokens of the page that belong to the sequence
  int64_t src;     // element offset of the first row
  bool ok;
};

// Tiles are numbered layer-major: CONTIG / RAGGED per (layer, head) then
// sequence then 128-key chunk; PAGED per layer then sequence then page.
__device__ __forceinline__ Tile decode(const Geom& g, int t) {
  Tile T;
  const int per = g.tile_prefix[g.batch];
  const int outer = t / per;
  const int r = t - outer * per;
  const int b = find_seq(g.tile_prefix, g.batch, r);
  const int j = r - g.tile_prefix[b];
  T.b = b;
  T.ok = true;
  if (g.layout == TRI_LAYOUT_PAGED) {
    T.l = outer;
    T.h = 0;
    T.i0 = j * g.block_size;
    T.rows = g.block_size * g.H;
    T.tvalid = min(g.block_size, g.len[b] - T.i0);
    const int blk = g.block_table[static_cast<int64_t>(b) * g.max_blocks + j];
    if (static_cast<unsigned>(blk) >= static_cast<unsigned>(g.num_blocks)) {
      T.ok = false;
      T.src = 0;
    } else {
      T.src = T.l * g.sL + static_cast<int64_t>(blk) * g.sB;
    }
  } else {
    T.l = outer / g.H;
    T.h = outer - T.l * g.H;
    T.i0 = j * kTileRows;
    T.rows = min(kTileRows, g.len[b] - T.i0);
    T.tvalid = T.rows;
    bool ok = true;
    T.src = row_elem(g, T.l, T.h, b, T.i0, &ok);
  }
  return T;
}

// Dot product of 8 bf16 (packed in x, element order) with 8 fp32 weights.
__device__ __forceinline__ float dot8(const uint4 x, const float (&w)[8]) {
  float a = __uint_as_float(x.x << 16) * w[0];
  a = fmaf(__uint_as_float(x.x & 0xffff0000u), w[1], a);
  a = fmaf(__uint_as_float(x.y << 16), w[2], a);
  a = fmaf(__uint_as_float(x.y & 0xffff0000u), w[3], a);
  a = fmaf(__uint_as_float(x.z << 16), w[4], a);
  a = fmaf(__uint_as_float(x.z & 0xffff0000u), w[5], a);
  a = fmaf(__uint_as_float(x.w << 16), w[6], a);
  a = fmaf(__uint_as_float(x.w & 0xffff0000u), w[7], a);
  return a;
}

__device__ __forceinline__ void load_w(const float* __restrict__ w, int lh, int l16, float (&wv)[8]) {
  const float4* p = reinterpret_cast<const float4*>(w + static_cast<int64_t>(lh) * kD + l16 * 8);
  const float4 a = __ldg(p), b = __ldg(p + 1);
  wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w;
  wv[4] = b.x; wv[5] = b.y; wv[6] = b.z; wv[7] = b.w;
}

__global__ void __launch_bounds__(kThreads, 1)
score_kernel(const __grid_constant__ Geom g, const float* __restrict__ w, float* __restrict__ scores,
             int ntiles) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(kStages) * kTileBytes);
  uint64_t* empty = full + kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one thread issues the bulk copies
    if (lane != 0) return;
    const uint64_t policy = policy_evict_first();
    int k = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
      const int s = k % kStages, n = k / kStages;
      if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) break;
      const Tile T = decode(g, t);
      if (T.ok) {
        const uint32_t bytes = static_cast<uint32_t>(T.rows) * kRowBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(smem + static_cast<size_t>(s) * kTileBytes, g.k + T.src, bytes, &full[s], policy);
      } else {
        flag(TRI_DEVFLAG_BAD_PAGE);
        mbar_arrive(&full[s]);
      }
    }
    // Never leave a copy in flight into shared memory of an exiting CTA:
    // wait (bounded) for the latest issue on every stage.
    for (int s = 0; s < kStages && s < k; ++s) {
      const int last = (k - 1 - s) / kStages;   // issues on stage s: s, s+S, ... < k
      mbar_wait_bounded(&full[s], last & 1);
    }
    return;
  }

  // ---------------- consumers
  const int half = lane >> 4, l16 = lane & 15;
  const int slot = warp * 2 + half;       // 0..15: which row of each 16-row group
  float wv[8];
  int cur_lh = -1;
  int k = 0;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
    const int s = k % kStages, n = k / kStages;
    if (!mbar_wait_bounded(&full[s], n & 1)) break;
    const Tile T = decode(g, t);
    if (T.ok) {
      const unsigned char* buf = smem + static_cast<size_t>(s) * kTileBytes + l16 * 16;
      int h, iters;
      float* out;
      if (g.layout == TRI_LAYOUT_PAGED) {
        h = slot % g.H;                                // fixed per half-warp: 16 % H == 0
        iters = (T.rows + 15) >> 4;
      } else {
        h = T.h;
        iters = (T.rows + 15) >> 4;
      }
      const int lh = T.l * g.H + h;
      if (lh != cur_lh) {
        load_w(w, lh, l16, wv);
        cur_lh = lh;
      }
      out = scores + (static_cast<int64_t>(lh) * g.batch + T.b) * g.score_stride + T.i0;

      uint4 x[kIters];
#pragma unroll
      for (int it = 0; it < kIters; ++it)
        if (it < iters) x[it] = *reinterpret_cast<const uint4*>(buf + (it * 16 + slot) * kRowBytes);
      float acc[kIters];
#pragma unroll
      for (int it = 0; it < kIters; ++it) acc[it] = it < iters ? dot8(x[it], wv) : 0.f;
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        if (it < iters) {    // warp-uniform
          float a = acc[it];
          a += __shfl_xor_sync(0xffffffffu, a, 8);
          a += __shfl_xor_sync(0xffffffffu, a, 4);
          a += __shfl_xor_sync(0xffffffffu, a, 2);
          a += __shfl_xor_sync(0xffffffffu, a, 1);
          const int r = it * 16 + slot;
          if (l16 == 0 && r < T.rows) {
            if (g.layout == TRI_LAYOUT_PAGED) {
              const int tok = r / g.H;
              if (tok < T.tvalid) out[tok] = a;
            } else {
              out[r] = a;
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
