// Max-over-offsets scoring on the tensor cores:
//     scores[u][i] = max_{t < |D|} sum_j w[l*H + h][t][j] * float(K_u[i][j]),
// w[.][t] being the (unaveraged) weight vector of offset t.
//
// Page "The future-offset average in TriAttention can be precomputed",
// section "What it saves, and what it does not": the fold relies on the
// average being linear; a maximum over the offsets does not fold, so each
// key needs one dot product per offset.  That is a skinny dense contraction
// [keys x 128] x [128 x |D|], which is what the tensor cores are for:
//  * warp 0 (one thread) streams 128-key tiles with 2-D TMA copies (two
//    64-element boxes, 128-byte swizzle: the canonical K-major operand
//    layout) into a ring of shared-memory stages;
//  * warp 1 (one thread) issues tcgen05.mma kind::f16 (M = 128 keys,
//    K = 16 per instruction) with the keys as A and the weights as B.  bf16
//    weights alone would cost 2^-9 of relative accuracy, so every weight is
//    split w = hi + lo into two bf16 parts (residual below 2^-16 of |w|); B
//    holds the hi rows and then the lo rows (N = 2 x |D| rounded up to 16),
//    so 8 MMAs per tile give both products in fp32 tensor-memory columns;
//    accumulators are double-buffered;
//  * warps 2-5 read the accumulator rows (tcgen05.ld, one key per thread),
//    add the hi and lo columns, take the max over the |D| offsets and store
//    the score.
// The weights of a (layer, head) are converted and swizzled into shared memory
// when a CTA's tile run reaches that head (runs are contiguous per CTA).
#pragma once

#include <cuda.h>
#include <cute/arch/mma_sm100_desc.hpp>

#include "common.cuh"
#include "score.cuh"

#ifndef TRI_SMAX_STAGES
#define TRI_SMAX_STAGES 4
#endif
#ifndef TRI_SMAX_MAX_OFFSETS
#define TRI_SMAX_MAX_OFFSETS 64
#endif
#ifndef TRI_SMAX_CTAS_PER_SM
#define TRI_SMAX_CTAS_PER_SM 1
#endif
#ifndef TRI_SMAX_ACC_BUFS
#define TRI_SMAX_ACC_BUFS 2
#endif


namespace tri {

// `raw` (a __shared__ array) advanced to the next multiple of kAlign bytes
// of the shared window, as the 128-byte swizzle of the TMA tiles needs.  The
// offset is added to the array pointer itself, so the compiler still sees a
// shared-memory pointer and emits shared loads; a round trip through an
// integer would leave a generic (64-bit) pointer, whose loads take the
// slower generic path and whose address arithmetic costs registers.
template <uint32_t kAlign>
__device__ __forceinline__ unsigned char* align_shared(unsigned char* raw) {
  static_assert((kAlign & (kAlign - 1)) == 0, "power of two");
  return raw + ((kAlign - (smem_addr(raw) & (kAlign - 1))) & (kAlign - 1));
}

namespace smax {

constexpr int kTileRows = score::kTileRows;     // 128 keys: the MMA's M
constexpr int kStages = TRI_SMAX_STAGES;
constexpr int kStageBytes = kTileRows * kRowBytes;   // 32 KB: two 16 KB boxes
constexpr int kBoxBytes = kStageBytes / 2;
constexpr int kMaxOffsets = TRI_SMAX_MAX_OFFSETS;
constexpr int kThreads = 6 * 32;
// The B operand holds each offset's weights twice, as bf16 hi rows
// [0, n_cols) and bf16 lo rows [n_cols, 2 n_cols), so one pass of 8 MMAs over
// a key tile (N = 2 n_cols) gives both partial products side by side, and the
// epilogue adds them.  (Accumulating hi and lo into the same columns took two
// passes, 16 MMAs of half the width per tile, and held the kernel at 5.6 TB/s
// with the key stream idle; the tensor pipe itself was 16 % busy.)
constexpr int kAccCols = 2 * kMaxOffsets;          // columns per accumulator buffer
// Accumulator buffers: the MMAs of a tile may run that many tiles ahead of
// the epilogue.
constexpr int kAccBufs = TRI_SMAX_ACC_BUFS;
constexpr uint32_t kTmemCols = kAccBufs * kAccCols;
static_assert(kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0, "tensor memory columns");
constexpr int kBBytesMax = 2 * kMaxOffsets * kRowBytes;   // hi and lo parts, N <= kMaxOffsets
constexpr size_t kBOffset = static_cast<size_t>(kStages) * kStageBytes;
constexpr size_t kBarOffset = kBOffset + kBBytesMax;
constexpr size_t kSmemBytes = kBarOffset + 256 + 1024;    // barriers, slot, alignment slack
static_assert((2 * kStages + 2 * kAccBufs) * 8 + 8 <= 256, "barrier area");

struct Args {
  const float* w;        // [L*H][n_offsets][128]
  float* scores;
  int ntiles;
  int n_offsets;         // 1 .. kMaxOffsets
  int n_cols;            // n_offsets rounded up to 16
};

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// A 5-D tiled load (the paged pool seen as [layer][page][token][head][128]).
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int x, int h, int t, int page,
                                            int layer, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(t), "r"(page), "r"(layer), "r"(smem_addr(bar)),
      "l"(policy)
      : "memory");
}

// A 128-key tile of one unit (l, h, b) of a PAGED cache: tiles are numbered
// per (layer, head), then sequence, then 128-key chunk (tile_prefix counts
// 128-key chunks per sequence); its keys are the pages p0 .. of sequence b.
struct HeadTile {
  int l, h, b, i0, rows;
  float* out;        // score of the tile's first key
};
__device__ __forceinline__ HeadTile head_tile(const Geom& g, int t, float* scores) {
  HeadTile T;
  const int per = g.tile_prefix[g.batch];
  const int lh = t / per, r = t - lh * per;
  T.b = find_seq(g.tile_prefix, g.batch, r);
  T.i0 = (r - g.tile_prefix[T.b]) * kTileRows;
  T.l = lh / g.H;
  T.h = lh - T.l * g.H;
  T.rows = min(kTileRows, g.len[T.b] - T.i0);
  T.out = scores + (static_cast<int64_t>(lh) * g.batch + T.b) * g.score_stride + T.i0;
  return T;
}

// K-major, 128-byte-swizzled operand: 8-row atoms of 1024 bytes (SBO), 16-byte
// units along K; version 1 for sm_100.
__device__ __forceinline__ uint64_t sw128_desc(const void* p) {
  cute::UMMA::SmemDescriptor d;
  d.desc_ = 0;
  d.version_ = 1;
  d.lbo_mode_ = 0;
  d.layout_type_ = static_cast<uint8_t>(cute::UMMA::LayoutType::SWIZZLE_128B);
  d.leading_byte_offset_ = 1;
  d.stride_byte_offset_ = 1024 >> 4;
  d.base_offset_ = 0;
  d.start_address_ = static_cast<uint16_t>((smem_addr(p) & 0x3ffffu) >> 4);
  return d.desc_;
}

// bf16 x bf16 -> fp32, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc(int n) {
  cute::UMMA::InstrDescriptor d;
  d.desc_ = 0;
  d.c_format_ = static_cast<uint8_t>(cute::UMMA::CFormat::F32);
  d.a_format_ = static_cast<uint8_t>(cute::UMMA::F16F32Format::BF16);
  d.b_format_ = static_cast<uint8_t>(cute::UMMA::F16F32Format::BF16);
  d.a_major_ = static_cast<uint8_t>(cute::UMMA::Major::K);
  d.b_major_ = static_cast<uint8_t>(cute::UMMA::Major::K);
  d.m_dim_ = kTileRows >> 4;
  d.n_dim_ = static_cast<uint8_t>(n >> 3);
  return d.desc_;
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  const uint32_t no_mask = 0u;    // no output lanes disabled
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(no_mask)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16 consecutive fp32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Byte offset of element (n, k) of a K-major operand with n_cols rows in two
// 64-element boxes, 128-byte swizzle: 16-byte chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(int n, int k, int n_cols) {
  const int box = k >> 6, kk = k & 63;
  return static_cast<uint32_t>(box * n_cols * 128 + (n >> 3) * 1024 + (n & 7) * 128 +
                               ((((kk >> 3) ^ (n & 7)) & 7) << 4) + (kk & 7) * 2);
}

__global__ void __launch_bounds__(kThreads, TRI_SMAX_CTAS_PER_SM)
score_max_kernel(const __grid_constant__ Geom g, const __grid_constant__ CUtensorMap kmap, const Args a) {
  extern __shared__ unsigned char smax_raw[];
  unsigned char* smem = align_shared<1024>(smax_raw);
  unsigned char* bsm = smem + kBOffset;               // B: hi rows, then lo rows
  const int n2 = 2 * a.n_cols;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + kAccBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // this CTA's contiguous run of tiles
  const int t_begin = static_cast<int>(static_cast<int64_t>(a.ntiles) * blockIdx.x / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(a.ntiles) * (blockIdx.x + 1) / gridDim.x);
  const int per_lh = g.tile_prefix[g.batch];          // tiles of one (layer, head)
  const uint32_t idesc = instr_desc(n2);
  const uint64_t policy = policy_evict_first();
  int k = 0, j = 0;                                   // stage-ring and accumulator counters
  for (int t0 = t_begin; t0 < t_end;) {
    const int lh = t0 / per_lh;
    const int t1 = min(t_end, (lh + 1) * per_lh);

    // weights of this head: bf16 hi / lo, swizzled (epilogue warps)
    if (warp >= 2) {
      const int kcol = threadIdx.x - 64;              // 0..127: one element column
      for (int n = 0; n < a.n_cols; ++n) {
        const float wv = n < a.n_offsets ? __ldg(a.w + (static_cast<int64_t>(lh) * a.n_offsets + n) * kD + kcol) : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(wv);
        const __nv_bfloat16 lo = __float2bfloat16_rn(wv - __bfloat162float(hi));
        *reinterpret_cast<__nv_bfloat16*>(bsm + sw128_offset(n, kcol, n2)) = hi;
        *reinterpret_cast<__nv_bfloat16*>(bsm + sw128_offset(a.n_cols + n, kcol, n2)) = lo;
      }
      fence_async_smem();
    }
    __syncthreads();

    if (warp == 0 && g.layout == TRI_LAYOUT_PAGED) {
      // ---------------- producer, PAGED: the whole warp, lane p on page p of
      // the tile (block_size is a power of two >= 8, so a tile is whole pages,
      // at most 16, and each page's rows are whole 1 KB swizzle atoms).  The
      // page ids of the next tile are loaded before this tile's slot is
      // awaited; pages outside the pool are left out.
      const int bs = g.block_size;
      auto page_of = [&](const HeadTile& T) -> int32_t {
        const int np = (T.rows + bs - 1) >> g.block_shift;
        return lane < np ? g.block_table[static_cast<int64_t>(T.b) * g.max_blocks + (T.i0 >> g.block_shift) + lane]
                         : -1;
      };
      HeadTile Tn;
      int32_t nxt = -1;
      if (t0 < t1) {
        Tn = head_tile(g, t0, a.scores);
        nxt = page_of(Tn);
      }
      for (int t = t0; t < t1; ++t, ++k) {
        const HeadTile T = Tn;
        const int32_t cur = nxt;
        if (t + 1 < t1) {
          Tn = head_tile(g, t + 1, a.scores);
          nxt = page_of(Tn);
        }
        const int s = k % kStages, n = k / kStages;
        int stop = 0;
        if (lane == 0) {
          if (n > 0 && !*abort_flag && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) *abort_flag = 1;
          stop = *abort_flag;
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) continue;
        const int np = (T.rows + bs - 1) >> g.block_shift;
        const bool valid = lane < np && static_cast<unsigned>(cur) < static_cast<unsigned>(g.num_blocks);
        const uint32_t ok = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) {
          if (ok != (1u << np) - 1u) flag(TRI_DEVFLAG_BAD_PAGE);
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(__popc(ok)) * bs * kRowBytes);
        }
        __syncwarp();                                 // the expected bytes are set before any copy lands
        if (valid) {
          unsigned char* stage = smem + static_cast<size_t>(s) * kStageBytes;
          const uint32_t off = static_cast<uint32_t>(lane * bs) * 128u;
          tma_load_5d(stage + off, &kmap, 0, T.h, 0, cur, T.l, &full[s], policy);
          tma_load_5d(stage + kBoxBytes + off, &kmap, 64, T.h, 0, cur, T.l, &full[s], policy);
        }
      }
    } else if (warp == 0) {
      // ---------------- producer, packed layouts: one thread
      if (lane == 0) {
        for (int t = t0; t < t1; ++t, ++k) {
          const int s = k % kStages, n = k / kStages;
          if (n > 0 && !*abort_flag && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) *abort_flag = 1;
          if (*abort_flag) continue;
          unsigned char* stage = smem + static_cast<size_t>(s) * kStageBytes;
          score::TileInfo T;
          int64_t src;
          bool ok;
          score::decode(g, t, a.scores, &T, &src, &ok);
          const int row = static_cast<int>(src / kD);
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(stage, &kmap, 0, row, &full[s], policy);
          tma_load_2d(stage + kBoxBytes, &kmap, 64, row, &full[s], policy);
        }
      } else {
        k += t1 - t0;
      }
    } else if (warp == 1) {
      // ---------------- MMA issue
      if (lane == 0) {
        for (int t = t0; t < t1; ++t, ++k, ++j) {
          const int s = k % kStages, n = k / kStages;
          const int ab = j % kAccBufs, na = j / kAccBufs;
          if (!*abort_flag && !mbar_wait_bounded(&full[s], n & 1)) *abort_flag = 1;
          if (!*abort_flag && na > 0 && !mbar_wait_bounded(&acc_empty[ab], (na - 1) & 1)) *abort_flag = 1;
          if (*abort_flag) continue;
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(ab * kAccCols);
          const unsigned char* stage = smem + static_cast<size_t>(s) * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t da = sw128_desc(stage + (kk >> 2) * kBoxBytes + (kk & 3) * 32);
            const uint64_t db = sw128_desc(bsm + (kk >> 2) * n2 * 128 + (kk & 3) * 32);
            mma_bf16(d_tmem, da, db, idesc, kk ? 1u : 0u);
          }
          mma_commit(&empty[s]);        // the stage is free once these MMAs have read it
          mma_commit(&acc_full[ab]);    // the accumulator is ready
        }
      } else {
        k += t1 - t0;
        j += t1 - t0;
      }
    } else {
      // ---------------- epilogue: one key per thread
      const int quarter = warp & 3;                   // tensor-memory lanes 32*quarter ..
      const int r = quarter * 32 + lane;
      for (int t = t0; t < t1; ++t, ++j) {
        const int ab = j % kAccBufs, na = j / kAccBufs;
        // the tile's output, decoded while the MMAs run (PAGED: keys in pages
        // outside the pool are not written)
        float* out;
        int rows;
        bool live;
        if (g.layout == TRI_LAYOUT_PAGED) {
          const HeadTile T = head_tile(g, t, a.scores);
          out = T.out;
          rows = T.rows;
          live = r < rows &&
                 static_cast<unsigned>(g.block_table[static_cast<int64_t>(T.b) * g.max_blocks +
                                                     ((T.i0 + r) >> g.block_shift)]) <
                     static_cast<unsigned>(g.num_blocks);
        } else {
          score::TileInfo T;
          int64_t src;
          bool ok;
          score::decode(g, t, a.scores, &T, &src, &ok);
          out = T.out;
          rows = T.rows;
          live = r < rows;
        }
        if (!*abort_flag && !mbar_wait_bounded(&acc_full[ab], na & 1)) *abort_flag = 1;
        if (*abort_flag) continue;
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * kAccCols);
        float best = 0.f;
        for (int c0 = 0; c0 < a.n_cols; c0 += 16) {  // 16 offsets at a time: hi + lo
          float sum[16], v[16];
          tmem_ld16(taddr + static_cast<uint32_t>(c0), sum);
          tmem_ld16(taddr + static_cast<uint32_t>(a.n_cols + c0), v);
#pragma unroll
          for (int i = 0; i < 16; ++i) sum[i] += v[i];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < a.n_offsets) best = c0 + i == 0 ? sum[i] : fmaxf(best, sum[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        if (live) out[r] = best;
      }
    }
    t0 = t1;
    __syncthreads();   // the next head's weights overwrite bhi / blo
  }

  // never exit with copies in flight (only possible after an abort)
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int s = 0; s < kStages && s < k; ++s) mbar_wait_bounded(&full[s], ((k - 1 - s) / kStages) & 1);
  }
  if (*abort_flag && threadIdx.x == 0) flag(TRI_DEVFLAG_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace smax
}  // namespace tri
