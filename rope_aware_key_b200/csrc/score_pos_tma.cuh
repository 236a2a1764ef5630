// The per-key-distance scorer (score_pos.cuh) for caches whose units are
// packed back to back (CONTIG and RAGGED with packed strides): one lane per
// key, every lane walking the 64 bands in the same order.
//
// That order is what makes it cheap:
//  * the band constants C_f are kernel parameters read at compile-time
//    offsets, so they are constant-bank operands of the integer multiplies
//    (no loads at all);
//  * the head's weights are the same for every lane of the tile, so each
//    16-byte shared load is a broadcast;
//  * the keys arrive by 2-D TMA in the 128-byte-swizzled layout (two boxes of
//    64 elements x 128 rows per tile), where chunk c of row r sits at chunk
//    c ^ (r mod 8): 32 lanes reading the same chunk of 32 rows hit all bank
//    groups, with no conflicts.
// Per key: 64 bands of packed f32x2 arithmetic, 16 shared loads of the key
// and 32 broadcast loads of weights.  A producer warp (one thread) streams the
// tiles, their weight rows and positions into a ring of stages; four
// consumer warps take one 128-key tile each time.
#pragma once

#include <cuda.h>

#include "score_max.cuh"
#include "score_pos.cuh"

#ifndef TRI_POST_STAGES
#define TRI_POST_STAGES 2
#endif
#ifndef TRI_POST_CTAS_PER_SM
#define TRI_POST_CTAS_PER_SM 3
#endif

namespace tri {
namespace score {

constexpr int kPtStages = TRI_POST_STAGES;
constexpr int kPtConsumerWarps = kTileRows / 32;             // one key per lane
constexpr int kPtThreads = (kPtConsumerWarps + 1) * 32;
constexpr int kPtBoxBytes = kTileBytes / 2;                  // 64 elements x 128 rows
constexpr size_t kPtPosOffset = static_cast<size_t>(kPtStages) * kTileBytes;
constexpr size_t kPtWOffset = kPtPosOffset + kPtStages * kPosStageBytes;
constexpr int kPtWBytes = kD * 4;
constexpr size_t kPtBarOffset = kPtWOffset + kPtStages * kPtWBytes;
constexpr size_t kPtInfoOffset = kPtBarOffset + 2 * kPtStages * sizeof(uint64_t);
constexpr size_t kPtSmemBytes = kPtInfoOffset + kPtStages * sizeof(TileInfo) + 1024;   // + alignment slack

// 16-byte chunk c (0..15) of row r of a stage: box c / 8, swizzled position.
__device__ __forceinline__ const uint4* sw_chunk(const unsigned char* stage, int r, int c) {
  return reinterpret_cast<const uint4*>(stage + (c >> 3) * kPtBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int PAIR>
__global__ void __launch_bounds__(kPtThreads, TRI_POST_CTAS_PER_SM)
score_pos_tma_kernel(const __grid_constant__ Geom g, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ Rot rot, const float* __restrict__ w, float* __restrict__ scores,
                     int ntiles) {
  extern __shared__ unsigned char pt_raw[];
  unsigned char* smem = align_shared<1024>(pt_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPtBarOffset);
  uint64_t* empty = full + kPtStages;
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + kPtInfoOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPtConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kPtConsumerWarps) {
    // ---------------- producer: one thread
    if (lane != 0) return;
    const uint64_t policy = policy_evict_first();
    int k = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
      const int s = k % kPtStages, n = k / kPtStages;
      if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) break;
      TileInfo T;
      int64_t src;
      bool ok;
      decode(g, t, scores, &T, &src, &ok);     // CONTIG / RAGGED: always ok
      T.tq = rot.qpos[T.b];
      info[s] = T;
      unsigned char* stage = smem + static_cast<size_t>(s) * kTileBytes;
      // a tiled copy always lands (and counts) the whole box; rows past the
      // unit belong to the next unit (or are zero-filled past the tensor)
      const uint32_t pbytes = rot.pos ? pos_row_bytes(T) : 0u;
      mbar_arrive_expect_tx(&full[s], kTileBytes + kPtWBytes + pbytes);
      const int row = static_cast<int>(src / kD);
      smax::tma_load_2d(stage, &kmap, 0, row, &full[s], policy);
      smax::tma_load_2d(stage + kPtBoxBytes, &kmap, 64, row, &full[s], policy);
      bulk_g2s(smem + kPtWOffset + s * kPtWBytes, w + static_cast<int64_t>(T.lh) * kD, kPtWBytes, &full[s], policy);
      if (rot.pos)
        copy_positions(rot.pos, scores, g.H, g.block_size, T, smem + kPtPosOffset + s * kPosStageBytes, &full[s],
                       policy);
    }
    for (int s = 0; s < kPtStages && s < k; ++s) mbar_wait_bounded(&full[s], ((k - 1 - s) / kPtStages) & 1);
    return;
  }

  // ---------------- consumers: lane = key
  const int r = warp * 32 + lane;
  int k = 0;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
    const int s = k % kPtStages, n = k / kPtStages;
    if (!mbar_wait_bounded(&full[s], n & 1)) break;
    const TileInfo T = info[s];
    const bool live = r < T.rows;
    const int32_t t_b = T.tq;
    const int32_t* sp = reinterpret_cast<const int32_t*>(smem + kPtPosOffset + s * kPosStageBytes);
    const int32_t p_i = !live ? t_b : rot.pos ? sp[r] : T.i0 + r;
    const Dist d = distance(t_b, p_i);
    const unsigned char* stage = smem + static_cast<size_t>(s) * kTileBytes;
    const float4* wr = reinterpret_cast<const float4*>(smem + kPtWOffset + s * kPtWBytes);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {          // bands 8j .. 8j + 7
      if constexpr (PAIR == 0) {
        // real parts: chunk j; imaginary parts: chunk j + 8
        const uint4 xr = *sw_chunk(stage, r, j);
        const uint4 xi = *sw_chunk(stage, r, j + 8);
        const float4 ar0 = wr[2 * j], ar1 = wr[2 * j + 1];
        const float4 ai0 = wr[16 + 2 * j], ai1 = wr[16 + 2 * j + 1];
        const float2 ar[4] = {make_float2(ar0.x, ar0.y), make_float2(ar0.z, ar0.w), make_float2(ar1.x, ar1.y),
                              make_float2(ar1.z, ar1.w)};
        const float2 ai[4] = {make_float2(ai0.x, ai0.y), make_float2(ai0.z, ai0.w), make_float2(ai1.x, ai1.y),
                              make_float2(ai1.z, ai1.w)};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int f = 8 * j + 2 * q;
          acc = band_pair(lo_hi(word(xr, q)), lo_hi(word(xi, q)), ar[q], ai[q], rot.c_hi[f], rot.c_lo[f],
                          rot.c_hi[f + 1], rot.c_lo[f + 1], d.D, d.sc, d.off, acc);
        }
      } else {
        // chunks 2j (bands 8j .. 8j+3) and 2j + 1 (8j+4 .. 8j+7), one (re, im) word per band
        const uint4 x0 = *sw_chunk(stage, r, 2 * j);
        const uint4 x1 = *sw_chunk(stage, r, 2 * j + 1);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 a = wr[4 * j + q];        // (re, im, re, im) of bands 8j + 2q, + 1
          const uint4& x = q < 2 ? x0 : x1;
          const uint32_t w0 = word(x, (2 * q) & 3), w1 = word(x, (2 * q + 1) & 3);
          const int f = 8 * j + 2 * q;
          acc = band_pair(lo_lo(w0, w1), hi_hi(w0, w1), make_float2(a.x, a.z), make_float2(a.y, a.w),
                          rot.c_hi[f], rot.c_lo[f], rot.c_hi[f + 1], rot.c_lo[f + 1], d.D, d.sc, d.off, acc);
        }
      }
    }
    if (live) {
      if (!d.in_range) flag(TRI_DEVFLAG_BAD_POSITION);
      T.out[r] = d.in_range ? -(acc.x + acc.y) : __int_as_float(0x7fc00000);   // -: the phase was shifted by pi
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace score
}  // namespace tri
