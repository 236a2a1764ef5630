// Scoring a pre-RoPE cache: every key carries its own distance to the query,
// Delta_i = t_b - p_i, and
//
//   scores[u][i] = Re sum_f a_f conj(k_f) e^{i omega_f Delta_i},
//
// with a_f the folded weight of the head (the offset mean W_f times E[q_f],
// written as w[re(f)] = Re a_f, w[im(f)] = Im a_f).  This is the averaging
// step of the page "The future-offset average in TriAttention can be
// precomputed" (section "The averaging step - the one we improve") with the
// kept distance taken per key instead of one scalar per pruning event.
//
// The keys stream through the same shared-memory ring as the folded scorer
// (score.cuh: one producer thread, bulk copies, full/empty barriers), and the
// tile's positions ride along on the same barrier, so that no consumer waits
// on a global load; only the consumers differ.  Eight lanes own a key, and the two chunks a lane
// reads hold 8 complete bands for either pairing.  Per band a lane needs cos
// and sin of omega_f * Delta_i:
//  * the phase is reduced exactly in integer arithmetic: with
//    C_f = omega_f / (2 pi) * 2^55 as an integer, bits 32..54 of
//    |Delta| * C_f (mod 2^64) are the first 23 bits of the fraction of a turn
//    of |Delta| omega_f / (2 pi); two integer multiplies give that word and
//    one logic op makes it the mantissa of m = 1 + fraction in [1, 2)
//    (truncation error < 2^-23 turn);
//  * one FMA maps m to phi = 2 pi m - 3 pi in [-pi, pi), exactly up to one
//    rounding, so phi is the phase minus pi (both sine and cosine change sign,
//    undone once per key); the sign of Delta goes into the FMA's constants;
//  * __sincosf (the hardware approximation) on [-pi, pi), where its absolute
//    error is about 4e-7.
// The phase error is therefore ~1.5e-6 rad at worst, which moves a score by
// at most that fraction of sum_f |a_f| |k_f|.
#pragma once

#include "score.cuh"

namespace tri {
namespace score {

constexpr int kBands = kD / 2;

// Per-call parameters of the distance scorer.
struct Rot {
  const int32_t* pos;            // positions, laid out like the scores; nullptr: p_i = i
  int32_t qpos[TRI_MAX_BATCH];   // query position t_b per sequence
  uint32_t c_hi[kBands];         // C_f = omega_f / (2 pi) * 2^55 (a 53-bit integer): high word
  uint32_t c_lo[kBands];         //                                                   low word
};

// One band's element of a 16-byte chunk of 8 bf16 (element order).
__device__ __forceinline__ float chunk_elem(const uint4 x, int e) {
  const uint32_t wd = e < 2 ? x.x : e < 4 ? x.y : e < 6 ? x.z : x.w;
  return (e & 1) ? __uint_as_float(wd & 0xffff0000u) : __uint_as_float(wd << 16);
}

// Eight lanes own a key: lane c8 = lane % 8 reads chunk c8 (slot 0) and
// chunk c8 + 8 (slot 1) of the row, 16 bytes each, so a key's eight lanes read
// 128 contiguous bytes per load and a warp's four keys fill the 32 banks once
// per 128 bytes (no conflicts).  Those two chunks hold 8 complete bands:
//   half-split:  lane band b = e:      re = (slot 0, e),  im = (slot 1, e),   f = 8 c8 + e
//   interleaved: lane band b = 4q + e: re = (slot q, 2e), im = (slot q, 2e+1), f = 4 (c8 + 8q) + e
template <int PAIR>
struct BandMap {
  static constexpr __device__ __forceinline__ int re_q(int b) { return PAIR == 0 ? 0 : b / 4; }
  static constexpr __device__ __forceinline__ int re_e(int b) { return PAIR == 0 ? b : 2 * (b % 4); }
  static constexpr __device__ __forceinline__ int im_q(int b) { return PAIR == 0 ? 1 : b / 4; }
  static constexpr __device__ __forceinline__ int im_e(int b) { return PAIR == 0 ? b : 2 * (b % 4) + 1; }
  static __device__ __forceinline__ int band(int b, int c8) {
    return PAIR == 0 ? 8 * c8 + b : 4 * (c8 + 8 * (b / 4)) + b % 4;
  }
};

// Shared memory of the distance scorer: the folded scorer's ring plus, per
// stage, the positions of the tile's keys (CONTIG / RAGGED: key r at r;
// PAGED: head h, token j at h * block_size + j), plus the lanes' band
// constants: entry (j, c8) = {C_hi, C_lo} of lane-local bands 2j and 2j + 1
// of lane c8, so that the eight lanes of a key read 128 contiguous bytes.
constexpr size_t kPosOffset = (kSmemBytes + 15) & ~size_t{15};
constexpr int kPosStageBytes = kTileRows * 4;
constexpr size_t kBandTabOffset = kPosOffset + kStages * kPosStageBytes;
constexpr size_t kPosSmemBytes = kBandTabOffset + 4 * 8 * 16;

// The positions of a tile, copied with it: one bulk copy per score row the
// tile touches (one, or H for a page), each rounded up to 4 entries (16
// bytes).  Rounding stays inside the row: a row holds the longest sequence
// rounded up to 4, and a tile starts at a multiple of 4 (128 keys, or a page
// of a multiple of 4 tokens -- checked on the host).
struct PosCopy {
  const int32_t* pos;
  const float* scores;
  unsigned char* buf;     // stage 0 of the positions area
  int H, block_size;
  __device__ __forceinline__ uint32_t row_bytes(const TileInfo& T) const {
    return static_cast<uint32_t>((T.paged ? T.tvalid : T.rows) + 3) / 4 * 16;
  }
  __device__ __forceinline__ uint32_t bytes(const TileInfo& T) const {
    return pos ? row_bytes(T) * (T.paged ? H : 1) : 0u;
  }
  __device__ __forceinline__ void issue(const TileInfo& T, int s, uint64_t* bar, uint64_t policy) const {
    if (!pos) return;
    const uint32_t nb = row_bytes(T);
    const int32_t* src = pos + (T.out - scores);
    unsigned char* dst = buf + s * kPosStageBytes;
    if (!T.paged) {
      bulk_g2s(dst, src, nb, bar, policy);
    } else {
      for (int h = 0; h < H; ++h)
        bulk_g2s(dst + h * block_size * 4, src + h * T.head_step, nb, bar, policy);
    }
  }
};

constexpr int kPosLanes = 8;                                   // lanes per key
constexpr int kPosRowsPerWarpPass = 32 / kPosLanes;            // 4 keys per warp per pass
constexpr int kPosGroup = kPosRowsPerWarpPass * kConsumerWarps;

// 2 pi with a zero last mantissa bit, so that 1.5 * k2Pi is a float too and
// fmaf(m, k2Pi, -1.5f * k2Pi) = k2Pi * (m - 1.5) up to one rounding.
__device__ __forceinline__ float two_pi_even() { return __uint_as_float(0x40c90fdau); }

template <int PAIR>
__global__ void __launch_bounds__(kThreads, TRI_SCORE_CTAS_PER_SM)
score_pos_kernel(const __grid_constant__ Geom g, const __grid_constant__ Rot rot, const float* __restrict__ w,
                 float* __restrict__ scores, int ntiles) {
  using M = BandMap<PAIR>;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + kInfoOffset);
  uint4* band_tab = reinterpret_cast<uint4*>(smem + kBandTabOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < 32) {
    const int j = threadIdx.x / kPosLanes, c = threadIdx.x % kPosLanes;
    const int f0 = M::band(2 * j, c), f1 = M::band(2 * j + 1, c);
    band_tab[threadIdx.x] = make_uint4(rot.c_hi[f0], rot.c_lo[f0], rot.c_hi[f1], rot.c_lo[f1]);
  }
  init_ring(full, empty);   // its barrier also publishes the table
  if (warp == kConsumerWarps) {
    if (lane == 0)
      produce(g, scores, smem, full, empty, info, ntiles,
              PosCopy{rot.pos, scores, smem + kPosOffset, g.H, g.block_size});
    return;
  }

  const int c8 = lane & (kPosLanes - 1);
  const int row0 = warp * kPosRowsPerWarpPass + lane / kPosLanes;
  // A lane's rows of a tile are row0 + 32 it.  PAGED rows interleave heads
  // (row = token * H + head, H | 8), so every row of the lane has head
  // row0 % H and the tokens advance by 32 / H per pass.
  const bool paged = g.layout == TRI_LAYOUT_PAGED;
  const int h0 = paged ? row0 % g.H : 0;
  const int tok0 = paged ? row0 / g.H : row0;
  const int tok_step = paged ? kPosGroup / g.H : kPosGroup;
  const float k2pi = two_pi_even();
  float wv[16];                                // the lane's two weight chunks, element order
  int cur_lh = -1;
  int k = 0;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
    const int s = k % kStages, n = k / kStages;
    if (!mbar_wait_bounded(&full[s], n & 1)) break;
    const TileInfo T = info[s];
    if (T.rows > 0) {
      const int lh = T.lh + h0;
      if (lh != cur_lh) {
        const float4* base = reinterpret_cast<const float4*>(w + static_cast<int64_t>(lh) * kD);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float4 a = __ldg(base + 2 * (c8 + 8 * q)), b = __ldg(base + 2 * (c8 + 8 * q) + 1);
          wv[8 * q + 0] = a.x; wv[8 * q + 1] = a.y; wv[8 * q + 2] = a.z; wv[8 * q + 3] = a.w;
          wv[8 * q + 4] = b.x; wv[8 * q + 5] = b.y; wv[8 * q + 6] = b.z; wv[8 * q + 7] = b.w;
        }
        cur_lh = lh;
      }
      const int32_t t_b = rot.qpos[T.b];
      const int32_t lim = t_b - 0x7fffffff;          // p < lim  <=>  t_b - p >= 2^31
      const int ntok = paged ? T.tvalid : T.rows;
      float* out = T.out + (paged ? h0 * T.head_step : 0);
      const int32_t* sp = reinterpret_cast<const int32_t*>(smem + kPosOffset + s * kPosStageBytes) +
                          (paged ? h0 * g.block_size : 0);
      const unsigned char* buf = smem + static_cast<size_t>(s) * kTileBytes + row0 * kRowBytes + c8 * 16;
      const int iters = (T.rows + kPosGroup - 1) / kPosGroup;
#pragma unroll 1
      for (int it = 0; it < iters; ++it) {   // warp-uniform
        const int tok = tok0 + it * tok_step;
        const bool live = tok < ntok;
        const int32_t p_i = !live ? t_b : rot.pos ? sp[tok] : T.i0 + tok;
        const bool in_range = p_i >= lim;
        // t_b - p_i in two's complement: exact when in range
        const uint32_t du = static_cast<uint32_t>(t_b) - static_cast<uint32_t>(p_i);
        const bool neg = static_cast<int32_t>(du) < 0;
        const uint32_t D = neg ? 0u - du : du;
        const float sc = neg ? -k2pi : k2pi;           // sin(-x) = -sin(x), cos(-x) = cos(x)
        const float off = -1.5f * sc;
        uint4 x[2];
        const unsigned char* rowp = buf + (live ? it * kPosGroup * kRowBytes : 0);
        x[0] = *reinterpret_cast<const uint4*>(rowp);
        x[1] = *reinterpret_cast<const uint4*>(rowp + 8 * 16);
        float part[2] = {0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 cc = band_tab[j * kPosLanes + c8];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int b = 2 * j + e;
            const float kr = chunk_elem(x[M::re_q(b)], M::re_e(b));
            const float ki = chunk_elem(x[M::im_q(b)], M::im_e(b));
            const float ar = wv[8 * M::re_q(b) + M::re_e(b)];
            const float ai = wv[8 * M::im_q(b) + M::im_e(b)];
            const float u = fmaf(ar, kr, ai * ki);        // Re a conj(k)
            const float v = fmaf(ai, kr, -(ar * ki));     // Im a conj(k)
            const uint32_t hi = e ? cc.z : cc.x, lo = e ? cc.w : cc.y;
            const uint32_t word = D * hi + __umulhi(D, lo);             // bits 32..63 of |Delta| C_f
            const float m = __uint_as_float((word & 0x007fffffu) | 0x3f800000u);
            const float phi = fmaf(m, sc, off);            // phase - pi, in [-pi, pi), signed like Delta
            float sn, cs;
            __sincosf(phi, &sn, &cs);
            part[e] = fmaf(u, cs, part[e]);
            part[e] = fmaf(-v, sn, part[e]);
          }
        }
        float a = part[0] + part[1];
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        a += __shfl_xor_sync(0xffffffffu, a, 4);
        if (c8 == 0 && live) {
          if (!in_range) flag(TRI_DEVFLAG_BAD_POSITION);
          out[tok] = in_range ? -a : __int_as_float(0x7fc00000);   // -: the phase was shifted by pi
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace score
}  // namespace tri
