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
// (score.cuh: one producer warp, bulk copies, full/empty barriers); the
// tile's positions and its heads' weight rows ride along on the same barrier,
// so no consumer waits on a global load.  This kernel takes every layout;
// score_pos_tma.cuh has a faster one for caches whose units are packed back
// to back.  Two lanes own a key, 32 bands each, in four steps of 8 bands; the
// band constants and the weights come from shared memory, laid out (or read
// in an order) that keeps the eight lanes of a quarter-warp on eight
// different bank groups; the complex products are packed f32x2 FMAs (two
// bands per instruction).  Per band a lane needs cos and sin of
// omega_f * Delta_i:
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

// Shared memory: the folded scorer's ring plus, per stage, the positions of
// the tile's keys (CONTIG / RAGGED: key r at r; PAGED: head h, token j at
// h * (tokens per tile) + j) and the weight rows of its heads (one, or H for a
// page), and once per CTA the band constants: for each group j of 8 bands
// {C_hi, C_lo} x 8 with a 16-byte pad, so that lanes reading eight different
// groups hit eight different bank groups.
constexpr size_t kPosOffset = (kSmemBytes + 15) & ~size_t{15};
constexpr int kPosStageBytes = kTileRows * 4;
constexpr size_t kWOffset = kPosOffset + kStages * kPosStageBytes;
constexpr int kMaxTileHeads = 8;                 // PAGED: H | 8
constexpr int kWStageBytes = kMaxTileHeads * kD * 4;
constexpr size_t kBandTabOffset = kWOffset + kStages * kWStageBytes;
constexpr int kBandTabStride = 8 * 8 + 16;
constexpr size_t kPosSmemBytes = kBandTabOffset + 8 * kBandTabStride;

// The positions of a tile: one bulk copy per score row the tile touches (one,
// or H for a page), each rounded up to 4 entries (16 bytes).  Rounding stays
// inside the row: a row holds the longest sequence rounded up to 4, and a
// tile starts at a multiple of 4 (128 keys, or a page of a multiple of 4
// tokens -- checked on the host).
__device__ __forceinline__ uint32_t pos_row_bytes(const TileInfo& T) {
  return static_cast<uint32_t>((T.paged ? T.tvalid : T.rows) + 3) / 4 * 16;
}
__device__ __forceinline__ void copy_positions(const int32_t* pos, const float* scores, int H, int tok_stride,
                                               const TileInfo& T, unsigned char* dst, uint64_t* bar,
                                               uint64_t policy) {
  const uint32_t nb = pos_row_bytes(T);
  const int32_t* src = pos + (T.out - scores);
  if (!T.paged) {
    bulk_g2s(dst, src, nb, bar, policy);
  } else {
    for (int h = 0; h < H; ++h) bulk_g2s(dst + h * tok_stride * 4, src + h * T.head_step, nb, bar, policy);
  }
}

// What travels with a tile besides its keys: its positions and the weight
// rows of its heads (consecutive rows of w).
struct PosCopy {
  const int32_t* pos;
  const float* scores;
  const float* w;
  unsigned char* smem;
  int H, tok_stride;      // PAGED: positions per head in a stage (tokens per tile)
  const int32_t* qpos;
  __device__ __forceinline__ void annotate(TileInfo& T) const { T.tq = qpos[T.b]; }
  __device__ __forceinline__ uint32_t w_bytes(const TileInfo& T) const {
    return static_cast<uint32_t>(T.paged ? H : 1) * kD * 4;
  }
  __device__ __forceinline__ uint32_t bytes(const TileInfo& T) const {
    return w_bytes(T) + (pos ? pos_row_bytes(T) * (T.paged ? H : 1) : 0u);
  }
  __device__ __forceinline__ void issue(const TileInfo& T, int s, uint64_t* bar, uint64_t policy) const {
    bulk_g2s(smem + kWOffset + s * kWStageBytes, w + static_cast<int64_t>(T.lh) * kD, w_bytes(T), bar, policy);
    if (pos) copy_positions(pos, scores, H, tok_stride, T, smem + kPosOffset + s * kPosStageBytes, bar, policy);
  }
};

// 2 pi with a zero last mantissa bit, so that 1.5 * k2Pi is a float too and
// fmaf(m, k2Pi, -1.5f * k2Pi) = k2Pi * (m - 1.5) up to one rounding.
__device__ __forceinline__ float two_pi_even() { return __uint_as_float(0x40c90fdau); }

__device__ __forceinline__ float2 lo_hi(uint32_t wd) {      // the two bf16 of a word, element order
  return make_float2(__uint_as_float(wd << 16), __uint_as_float(wd & 0xffff0000u));
}
__device__ __forceinline__ float2 lo_lo(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a << 16), __uint_as_float(b << 16));
}
__device__ __forceinline__ float2 hi_hi(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u));
}
__device__ __forceinline__ uint32_t word(const uint4& x, int i) { return i == 0 ? x.x : i == 1 ? x.y : i == 2 ? x.z : x.w; }

// Two bands (the x and y halves) of one key, added into acc:
//   Re a conj(k) e^{i phi'} = cos phi' (a_r k_r + a_i k_i) + sin phi' (a_r k_i - a_i k_r)
// with phi' the phase minus pi, built from the bits of |Delta| C_f (see the
// top of the file).  The two products of the key and the weight do not
// depend on the phase, so they are formed while the sine and cosine are in
// flight, and one packed FMA each then adds them in: six packed operations
// for the two bands.
__device__ __forceinline__ float2 band_pair(float2 kr, float2 ki, float2 ar, float2 ai, uint32_t hi0, uint32_t lo0,
                                            uint32_t hi1, uint32_t lo1, uint32_t D, float2 sc, float2 off,
                                            float2 acc) {
  const uint32_t w0 = D * hi0 + __umulhi(D, lo0);
  const uint32_t w1 = D * hi1 + __umulhi(D, lo1);
  const float2 m = make_float2(__uint_as_float((w0 & 0x007fffffu) | 0x3f800000u),
                               __uint_as_float((w1 & 0x007fffffu) | 0x3f800000u));
  const float2 phi = __ffma2_rn(m, sc, off);
  float2 sn, cs;
  __sincosf(phi.x, &sn.x, &cs.x);
  __sincosf(phi.y, &sn.y, &cs.y);
  const float2 P = __ffma2_rn(ar, kr, __fmul2_rn(ai, ki));                          // a_r k_r + a_i k_i
  const float2 Q = __ffma2_rn(ar, ki, __fmul2_rn(make_float2(-ai.x, -ai.y), kr));   // a_r k_i - a_i k_r
  acc = __ffma2_rn(cs, P, acc);
  return __ffma2_rn(sn, Q, acc);
}

// Per-key distance terms shared by the scorers: whether t_b - p_i is in
// range, |t_b - p_i|, and the FMA constants that put its sign into the phase.
struct Dist {
  uint32_t D;
  float2 sc, off;
  bool in_range;
};
__device__ __forceinline__ Dist distance(int32_t t_b, int32_t p_i) {
  Dist d;
  d.in_range = p_i >= t_b - 0x7fffffff;                      // t_b - p_i < 2^31 (t_b >= 0)
  const uint32_t du = static_cast<uint32_t>(t_b) - static_cast<uint32_t>(p_i);   // exact when in range
  const bool neg = static_cast<int32_t>(du) < 0;
  d.D = neg ? 0u - du : du;
  const float sc = neg ? -two_pi_even() : two_pi_even();     // sin(-x) = -sin(x), cos(-x) = cos(x)
  d.sc = make_float2(sc, sc);
  d.off = make_float2(-1.5f * sc, -1.5f * sc);
  return d;
}

// Band f of band group j, slot e (8 bands per group): f = 8 j + e for both
// pairings.  Half split: re(f) = f, im(f) = f + 64, so group j is chunk j
// (real parts) and chunk j + 8 (imaginary parts).  Interleaved: re(f) = 2f,
// im(f) = 2f + 1, so group j is chunks 2j and 2j + 1.
constexpr int kPosLanes = 2;                                    // lanes per key
constexpr int kPosKeysPerWarp = 32 / kPosLanes;
static_assert(kPosKeysPerWarp * kConsumerWarps == kTileRows, "one key per lane pair per tile");

template <int PAIR>
__global__ void __launch_bounds__(kThreads, TRI_SCORE_CTAS_PER_SM)
score_pos_kernel(const __grid_constant__ Geom g, const __grid_constant__ Rot rot, const float* __restrict__ w,
                 float* __restrict__ scores, int ntiles) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + kInfoOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < kBands) {   // band f -> group f / 8, slot f % 8
    uint2* tab = reinterpret_cast<uint2*>(smem + kBandTabOffset + (threadIdx.x / 8) * kBandTabStride);
    tab[threadIdx.x % 8] = make_uint2(rot.c_hi[threadIdx.x], rot.c_lo[threadIdx.x]);
  }
  init_ring(full, empty);   // its barrier also publishes the table
  if (warp == kConsumerWarps) {
    produce(g, scores, smem, full, empty, info, blockIdx.x, ntiles, gridDim.x,
            PosCopy{rot.pos, scores, w, smem, g.H, g.block_size * g.pages_per_tile, rot.qpos});
    return;
  }

  // This lane's key in every tile, and which half of its bands (groups
  // 4 hf .. 4 hf + 3).  Lane pairs start their groups at different offsets,
  // so the eight lanes of a quarter-warp take eight different groups at
  // every step; lanes of the upper half read their second 16 bytes first,
  // which puts them on the other four bank groups.
  const int r = warp * kPosKeysPerWarp + (lane >> 1);
  const int hf = lane & 1;
  const int start = (lane >> 1) & 3;
  const bool paged = g.layout == TRI_LAYOUT_PAGED;
  const int h = paged ? r % g.H : 0;               // PAGED rows interleave heads: row = token * H + head
  const int tok = paged ? r / g.H : r;
  const int tok_stride = g.block_size * g.pages_per_tile;   // PAGED: positions per head in a stage
  int k = 0;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
    const int s = k % kStages, n = k / kStages;
    if (!mbar_wait_bounded(&full[s], n & 1)) break;
    const TileInfo T = info[s];
    const bool live = r < T.rows && tok < (paged ? T.tvalid : T.rows) &&
                      (!paged || ((T.page_ok >> (tok / g.block_size)) & 1u));
    if (T.rows > 0) {
      const int32_t t_b = T.tq;
      const int32_t* sp = reinterpret_cast<const int32_t*>(smem + kPosOffset + s * kPosStageBytes);
      const int32_t p_i = !live ? t_b : rot.pos ? sp[paged ? h * tok_stride + tok : r] : T.i0 + tok;
      const Dist d = distance(t_b, p_i);
      const unsigned char* row = smem + static_cast<size_t>(s) * kTileBytes + (live ? r : 0) * kRowBytes;
      const float* wr = reinterpret_cast<const float*>(smem + kWOffset + s * kWStageBytes) + h * kD;
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = 4 * hf + ((c + start) & 3);
        const uint4* tab = reinterpret_cast<const uint4*>(smem + kBandTabOffset + j * kBandTabStride);
        if constexpr (PAIR == 0) {
          uint4 cst[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) cst[q] = tab[q];              // {hi, lo} of slots 2q, 2q + 1
          const uint4 xr = *reinterpret_cast<const uint4*>(row + j * 16);
          const uint4 xi = *reinterpret_cast<const uint4*>(row + (j + 8) * 16);
          // 16-byte halves in the order (hf, 1 - hf)
          const float4 aA = *reinterpret_cast<const float4*>(wr + 8 * j + 4 * hf);
          const float4 aB = *reinterpret_cast<const float4*>(wr + 8 * j + 4 * (1 - hf));
          const float4 iA = *reinterpret_cast<const float4*>(wr + 64 + 8 * j + 4 * hf);
          const float4 iB = *reinterpret_cast<const float4*>(wr + 64 + 8 * j + 4 * (1 - hf));
          const float4 ar0 = hf ? aB : aA, ar1 = hf ? aA : aB;
          const float4 ai0 = hf ? iB : iA, ai1 = hf ? iA : iB;
          const float2 ar[4] = {make_float2(ar0.x, ar0.y), make_float2(ar0.z, ar0.w), make_float2(ar1.x, ar1.y),
                                make_float2(ar1.z, ar1.w)};
          const float2 ai[4] = {make_float2(ai0.x, ai0.y), make_float2(ai0.z, ai0.w), make_float2(ai1.x, ai1.y),
                                make_float2(ai1.z, ai1.w)};
#pragma unroll
          for (int q = 0; q < 4; ++q)   // slots 2q, 2q + 1: word q of each chunk
            acc = band_pair(lo_hi(word(xr, q)), lo_hi(word(xi, q)), ar[q], ai[q], cst[q].x, cst[q].y, cst[q].z,
                            cst[q].w, d.D, d.sc, d.off, acc);
        } else {
          // chunk 2j holds slots 0..3, chunk 2j+1 slots 4..7, one (re, im) word
          // each; upper-half lanes take the second chunk first (bank spread)
          const uint4 x0 = *reinterpret_cast<const uint4*>(row + (2 * j + hf) * 16);
          const uint4 x1 = *reinterpret_cast<const uint4*>(row + (2 * j + 1 - hf) * 16);
          const float4* wq = reinterpret_cast<const float4*>(wr + 16 * j);   // (re, im, re, im) per float4
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // slots 2qq, 2qq + 1
            const int qq = q ^ (2 * hf);
            const float4 aq = wq[qq];
            const uint4 cq = tab[qq];
            const uint4& x = q < 2 ? x0 : x1;
            const uint32_t w0 = word(x, (2 * q) & 3), w1 = word(x, (2 * q + 1) & 3);
            acc = band_pair(lo_lo(w0, w1), hi_hi(w0, w1), make_float2(aq.x, aq.z), make_float2(aq.y, aq.w), cq.x,
                            cq.y, cq.z, cq.w, d.D, d.sc, d.off, acc);
          }
        }
      }
      float a = acc.x + acc.y;
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      if (hf == 0 && live) {
        if (!d.in_range) flag(TRI_DEVFLAG_BAD_POSITION);
        // minus: the phase was shifted by pi
        T.out[paged ? static_cast<int64_t>(h) * T.head_step + tok : tok] =
            d.in_range ? -a : __int_as_float(0x7fc00000);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace score
}  // namespace tri
