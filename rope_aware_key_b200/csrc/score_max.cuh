// Max-over-offsets scoring on the tensor cores:
//     scores[u][i] = max_{t < |D|} sum_j w[l*H + h][t][j] * float(K_u[i][j]),
// w[.][t] being the (unaveraged) weight vector of offset t.
//
// Page "The future-offset average in TriAttention can be precomputed",
// section "What it saves, and what it does not": the fold relies on the
// average being linear; a maximum over the offsets does not fold, so each
// key needs one dot product per offset.  That is a skinny dense contraction
// [keys x 128] x [128 x |D|], which is what the tensor cores are for:
//  * warp 0 streams 128-key tiles with TMA copies (two 64-element boxes,
//    128-byte swizzle: the canonical K-major operand layout) into a ring of
//    shared-memory stages: one thread and 2-D copies for packed layouts, a
//    lane per page and 5-D copies for paged pools;
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
// The weights of a (layer, head), or of all heads of a layer for whole-page
// paged tiles, are converted and swizzled into shared memory when a CTA's
// tile run reaches them (runs are contiguous per CTA).
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
// The B operand holds each offset's weights twice, as a bf16 hi row and the
// bf16 lo row after it (offset n: rows 2n and 2n + 1 of its head's block of
// head_cols = 2 |D| rounded up to 16 rows), so one pass of 8 MMAs over a key
// tile gives both partial products in adjacent columns, and the epilogue adds
// each pair.  (Accumulating hi and lo into the same columns took two passes,
// 16 MMAs of half the width per tile, and held the kernel at 5.6 TB/s with
// the key stream idle; the tensor pipe itself was 16 % busy.)
// With a PAGED cache whose heads fit one MMA (H * head_cols <= 256), B holds
// the weights of every head of the layer (head h: rows h * head_cols ..) and
// a tile is whole pages of all heads, one box pair per page, each page laid
// head-major in the stage; every key's accumulator row then carries every
// head's columns.  A warp's 32 rows hold one head, or 32 / block_size heads,
// and the warp reads only those heads' columns.
constexpr int kMaxB = 256;                         // B rows: heads * head_cols <= the MMA's largest N
constexpr int kAccCols = kMaxB;                    // columns per accumulator buffer
// Accumulator buffers: the MMAs of a tile may run that many tiles ahead of
// the epilogue.
constexpr int kAccBufs = TRI_SMAX_ACC_BUFS;
constexpr uint32_t kTmemCols = kAccBufs * kAccCols;
// Warps: 0 producer, 1 MMA issue, then one epilogue warpgroup per accumulator
// buffer (tile t of a CTA's walk goes to buffer and warpgroup t mod kAccBufs),
// so the epilogue works on kAccBufs tiles at once.
constexpr int kEpiWarps = 4 * kAccBufs;
constexpr int kThreads = (2 + kEpiWarps) * 32;
static_assert(kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0, "tensor memory columns");
constexpr int kBBytesMax = kMaxB * kRowBytes;             // hi and lo parts of every head in B
constexpr size_t kBOffset = static_cast<size_t>(kStages) * kStageBytes;
constexpr size_t kBarOffset = kBOffset + kBBytesMax;
// PAGED: page ids of the producer's next tiles, [2][kIdTiles][kMaxPages]
constexpr int kIdTiles = 32;                              // tiles decoded at once, a lane each
constexpr int kMaxPages = 16;                             // pages of a tile: 128 rows of >= 8 per page
constexpr size_t kIdsOffset = kBarOffset + 256;
constexpr size_t kSmemBytes = kIdsOffset + 2 * kIdTiles * kMaxPages * 4 + 1024;   // + alignment slack
static_assert((2 * kStages + 2 * kAccBufs) * 8 + 8 <= 256, "barrier area");

struct Args {
  const float* w;        // [L*H][n_offsets][128]
  float* scores;
  int ntiles;
  int n_offsets;         // 1 .. kMaxOffsets
  int head_cols;         // B rows (accumulator columns) per head: 2 n_offsets rounded up to 16
  int heads;             // heads in B: 1, or H for whole-page PAGED tiles
  int head_shift;        // log2(heads)
  int whole_pages;       // PAGED: tiles of whole pages of all heads (else of one head)
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

// A 5-D tiled load from a paged pool: coordinates (element, c1, c2, page,
// layer), c1 / c2 the head / token (one-head map) or token / head (all-heads
// map).
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int x, int c1, int c2, int page,
                                            int layer, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(c1), "r"(c2), "r"(page), "r"(layer), "r"(smem_addr(bar)),
      "l"(policy)
      : "memory");
}

// Tiles are numbered outer index (a weight run), then sequence, then chunk
// of the sequence; tile_prefix counts each sequence's chunks.  A CTA walks a
// contiguous range of tiles, so the walk keeps (outer, b, j) and steps it,
// searching tile_prefix only for the range's first tile.
struct Cursor {
  int outer, b, j;
};
__device__ __forceinline__ Cursor cursor_at(const Geom& g, int t) {
  Cursor c;
  const int per = g.tile_prefix[g.batch];
  c.outer = t / per;
  const int r = t - c.outer * per;
  c.b = find_seq(g.tile_prefix, g.batch, r);
  c.j = r - g.tile_prefix[c.b];
  return c;
}
// The next tile (one must exist: sequences without tiles are passed over).
__device__ __forceinline__ void cursor_next(const Geom& g, Cursor& c) {
  ++c.j;
  while (c.j >= g.tile_prefix[c.b + 1] - g.tile_prefix[c.b]) {
    c.j = 0;
    if (++c.b == g.batch) {
      c.b = 0;
      ++c.outer;
    }
  }
}

// A 128-key tile of a packed layout (CONTIG / RAGGED): chunk j of unit
// (outer = l*H + h, b).
struct PackedTile {
  int rows;          // keys of the tile inside the sequence
  int row;           // key row of the tile's first key in the [rows][128] view
  float* out;        // score of the tile's first key
};
__device__ __forceinline__ PackedTile packed_tile(const Geom& g, const Cursor& c, float* scores) {
  PackedTile T;
  const int l = c.outer / g.H, h = c.outer - l * g.H;
  const int i0 = c.j * kTileRows;
  T.rows = min(kTileRows, g.len[c.b] - i0);
  bool ok = true;
  T.row = static_cast<int>(row_elem(g, l, h, c.b, i0, &ok) / kD);
  T.out = scores + (static_cast<int64_t>(c.outer) * g.batch + c.b) * g.score_stride + i0;
  return T;
}

// A tile of a PAGED cache, in one of two forms:
//  * whole pages (Args::whole_pages): pages_per_tile consecutive pages of
//    sequence b in layer l = outer, all heads, each page head-major in the
//    stage;
//  * one head: 128 consecutive keys of unit (l, h, b), outer = l*H + h, a
//    page's rows of that head after another's.
struct PagedTile {
  int l, h;          // layer; head (one-head tiles) or 0
  int np;            // pages in the tile
  int64_t tbl;       // block-table index of the tile's first page
  int tvalid;        // tokens of the tile inside the sequence
  float* out;        // score of the tile's first token (of head h, or of head 0)
};
__device__ __forceinline__ PagedTile paged_tile(const Geom& g, const Cursor& c, bool whole, float* scores) {
  PagedTile T;
  const int span = whole ? g.pages_per_tile << g.block_shift : kTileRows;
  T.l = whole ? c.outer : c.outer / g.H;
  T.h = whole ? 0 : c.outer - T.l * g.H;
  const int i0 = c.j * span;
  T.tvalid = min(span, g.len[c.b] - i0);
  T.np = (T.tvalid + g.block_size - 1) >> g.block_shift;
  T.tbl = static_cast<int64_t>(c.b) * g.max_blocks + (i0 >> g.block_shift);
  T.out = scores + (static_cast<int64_t>(T.l * g.H + T.h) * g.batch + c.b) * g.score_stride + i0;
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

// Consecutive fp32 columns at ta (as many as x holds) and at tb (as many as
// y holds) of this warp's 32 tensor-memory lanes, one lane per thread: both
// loads are issued and then awaited once, inside one asm statement, so no use
// of the registers can be scheduled ahead of the wait.  Callers start every
// load of 32 columns on a multiple of 32 and every load of 16 on a multiple
// of 16.
__device__ __forceinline__ void tmem_ld_pair(uint32_t ta, uint32_t tb, uint32_t (&x)[32], uint32_t (&y)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, "
      "%20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31"
      "}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, "
      "%50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63"
      "}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
        "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15]),
        "=r"(x[16]), "=r"(x[17]), "=r"(x[18]), "=r"(x[19]), "=r"(x[20]), "=r"(x[21]), "=r"(x[22]), "=r"(x[23]),
        "=r"(x[24]), "=r"(x[25]), "=r"(x[26]), "=r"(x[27]), "=r"(x[28]), "=r"(x[29]), "=r"(x[30]), "=r"(x[31]),
        "=r"(y[0]), "=r"(y[1]), "=r"(y[2]), "=r"(y[3]), "=r"(y[4]), "=r"(y[5]), "=r"(y[6]), "=r"(y[7]),
        "=r"(y[8]), "=r"(y[9]), "=r"(y[10]), "=r"(y[11]), "=r"(y[12]), "=r"(y[13]), "=r"(y[14]), "=r"(y[15]),
        "=r"(y[16]), "=r"(y[17]), "=r"(y[18]), "=r"(y[19]), "=r"(y[20]), "=r"(y[21]), "=r"(y[22]), "=r"(y[23]),
        "=r"(y[24]), "=r"(y[25]), "=r"(y[26]), "=r"(y[27]), "=r"(y[28]), "=r"(y[29]), "=r"(y[30]), "=r"(y[31])
      : "r"(ta), "r"(tb)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_pair(uint32_t ta, uint32_t tb, uint32_t (&x)[16], uint32_t (&y)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15"
      "}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31"
      "}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
        "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15]),
        "=r"(y[0]), "=r"(y[1]), "=r"(y[2]), "=r"(y[3]), "=r"(y[4]), "=r"(y[5]), "=r"(y[6]), "=r"(y[7]),
        "=r"(y[8]), "=r"(y[9]), "=r"(y[10]), "=r"(y[11]), "=r"(y[12]), "=r"(y[13]), "=r"(y[14]), "=r"(y[15])
      : "r"(ta), "r"(tb)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_pair(uint32_t ta, uint32_t tb, uint32_t (&x)[32], uint32_t (&y)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, "
      "%20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31"
      "}, [%48];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47"
      "}, [%49];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
        "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15]),
        "=r"(x[16]), "=r"(x[17]), "=r"(x[18]), "=r"(x[19]), "=r"(x[20]), "=r"(x[21]), "=r"(x[22]), "=r"(x[23]),
        "=r"(x[24]), "=r"(x[25]), "=r"(x[26]), "=r"(x[27]), "=r"(x[28]), "=r"(x[29]), "=r"(x[30]), "=r"(x[31]),
        "=r"(y[0]), "=r"(y[1]), "=r"(y[2]), "=r"(y[3]), "=r"(y[4]), "=r"(y[5]), "=r"(y[6]), "=r"(y[7]),
        "=r"(y[8]), "=r"(y[9]), "=r"(y[10]), "=r"(y[11]), "=r"(y[12]), "=r"(y[13]), "=r"(y[14]), "=r"(y[15])
      : "r"(ta), "r"(tb)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_pair(uint32_t ta, uint32_t tb, uint32_t (&x)[16], uint32_t (&y)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15"
      "}, [%48];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, "
      "%34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47"
      "}, [%49];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
        "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15]),
        "=r"(y[0]), "=r"(y[1]), "=r"(y[2]), "=r"(y[3]), "=r"(y[4]), "=r"(y[5]), "=r"(y[6]), "=r"(y[7]),
        "=r"(y[8]), "=r"(y[9]), "=r"(y[10]), "=r"(y[11]), "=r"(y[12]), "=r"(y[13]), "=r"(y[14]), "=r"(y[15]),
        "=r"(y[16]), "=r"(y[17]), "=r"(y[18]), "=r"(y[19]), "=r"(y[20]), "=r"(y[21]), "=r"(y[22]), "=r"(y[23]),
        "=r"(y[24]), "=r"(y[25]), "=r"(y[26]), "=r"(y[27]), "=r"(y[28]), "=r"(y[29]), "=r"(y[30]), "=r"(y[31])
      : "r"(ta), "r"(tb)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_one(uint32_t ta, uint32_t (&x)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15"
      "}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
        "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15])
      : "r"(ta)
      : "memory");
}

// Byte offset of element (n, k) of a K-major operand with n_rows rows in two
// 64-element boxes, 128-byte swizzle: 16-byte chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(int n, int k, int n_rows) {
  const int box = k >> 6, kk = k & 63;
  return static_cast<uint32_t>(box * n_rows * 128 + (n >> 3) * 1024 + (n & 7) * 128 +
                               ((((kk >> 3) ^ (n & 7)) & 7) << 4) + (kk & 7) * 2);
}

__global__ void __launch_bounds__(kThreads, TRI_SMAX_CTAS_PER_SM)
score_max_kernel(const __grid_constant__ Geom g, const __grid_constant__ CUtensorMap kmap, const Args a) {
  extern __shared__ unsigned char smax_raw[];
  unsigned char* smem = align_shared<1024>(smax_raw);
  unsigned char* bsm = smem + kBOffset;               // B: per head, hi rows then lo rows
  const int n2 = a.heads * a.head_cols;
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
  const int per_run = g.tile_prefix[g.batch];         // tiles of one weight run: (layer, head), or a layer
  const uint32_t idesc = instr_desc(n2);
  const uint64_t policy = policy_evict_first();
  int k = 0, j = 0;                                   // stage-ring and accumulator counters
  int j_last = -1;                                    // MMA thread: the last tile whose MMAs it committed
  for (int t0 = t_begin; t0 < t_end;) {
    const int run = t0 / per_run;
    const int t1 = min(t_end, (run + 1) * per_run);

    // weights of this run's heads: bf16 hi / lo, swizzled (epilogue warps)
    if (warp >= 2) {
      const int kcol = (threadIdx.x - 64) & (kD - 1);   // one element column
      const int part = (threadIdx.x - 64) / kD;         // the warpgroups share the offsets
      const int per_head = a.head_cols >> 1;          // offset slots per head (the last ones zero)
      for (int m = part; m < a.heads * per_head; m += kAccBufs) {
        const int hh = m / per_head, n = m - hh * per_head;
        const int64_t lh = static_cast<int64_t>(run) * a.heads + hh;
        const float wv = n < a.n_offsets ? __ldg(a.w + (lh * a.n_offsets + n) * kD + kcol) : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(wv);
        const __nv_bfloat16 lo = __float2bfloat16_rn(wv - __bfloat162float(hi));
        const int row = hh * a.head_cols + 2 * n;
        *reinterpret_cast<__nv_bfloat16*>(bsm + sw128_offset(row, kcol, n2)) = hi;
        *reinterpret_cast<__nv_bfloat16*>(bsm + sw128_offset(row + 1, kcol, n2)) = lo;
      }
      fence_async_smem();
    }
    __syncthreads();

    if (warp == 0 && g.layout == TRI_LAYOUT_PAGED) {
      // ---------------- producer, PAGED: the whole warp.  Lane i decodes
      // tile tc + i of a group of 32 and loads its page ids (the pages of a
      // tile are at most 16: block_size is a power of two, a page's rows fill
      // whole 1 KB swizzle atoms and a tile is whole pages) while the previous
      // group's copies are issued; each group's ids go to shared memory.  Per
      // tile, lane p copies page p; pages outside the pool are left out.
      const bool whole = a.whole_pages != 0;
      const uint32_t page_rows = static_cast<uint32_t>(g.block_size) << a.head_shift;
      int32_t* ids = reinterpret_cast<int32_t*>(smem + kIdsOffset);
      int32_t v[kMaxPages];
      auto fetch = [&](int tc, int& l_, int& h_, int& np_) {
        const int ti = tc + lane;
        l_ = h_ = np_ = 0;
        if (ti < t1) {
          const PagedTile T = paged_tile(g, cursor_at(g, ti), whole, a.scores);
          l_ = T.l;
          h_ = T.h;
          np_ = T.np;
#pragma unroll
          for (int p = 0; p < kMaxPages; ++p) v[p] = p < np_ ? g.block_table[T.tbl + p] : -1;
        } else {
#pragma unroll
          for (int p = 0; p < kMaxPages; ++p) v[p] = -1;     // past the range: no pages
        }
      };
      auto stash = [&](int buf) {
#pragma unroll
        for (int p = 0; p < kMaxPages; ++p) ids[(buf * kIdTiles + lane) * kMaxPages + p] = v[p];
      };
      int cl, ch, cnp;
      fetch(t0, cl, ch, cnp);
      stash(0);
      __syncwarp();
      for (int tc = t0, buf = 0; tc < t1; tc += kIdTiles, buf ^= 1) {
        const bool more = tc + kIdTiles < t1;
        int nl = 0, nh = 0, nnp = 0;
        if (more) fetch(tc + kIdTiles, nl, nh, nnp);    // in flight while this group is issued
        const int nt = min(kIdTiles, t1 - tc);
        for (int i = 0; i < nt; ++i, ++k) {
          const int l = __shfl_sync(0xffffffffu, cl, i), h = __shfl_sync(0xffffffffu, ch, i);
          const int np = __shfl_sync(0xffffffffu, cnp, i);
          const int32_t cur = lane < np ? ids[(buf * kIdTiles + i) * kMaxPages + lane] : -1;
#ifdef TRI_TEST_HOOKS
          if (tc + i == g.test_skip_tile) continue;   // test builds: no copy and no arrival for this tile
#endif
          const int s = k % kStages, n = k / kStages;
          int stop = 0;
          if (lane == 0) {
            if (n > 0 && !*abort_flag && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) *abort_flag = 1;
            stop = *abort_flag;
          }
          if (__shfl_sync(0xffffffffu, stop, 0)) continue;
          const bool valid = lane < np && static_cast<unsigned>(cur) < static_cast<unsigned>(g.num_blocks);
          const uint32_t ok = __ballot_sync(0xffffffffu, valid);
          if (lane == 0) {
            if (ok != (1u << np) - 1u) flag(TRI_DEVFLAG_BAD_PAGE);
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(__popc(ok)) * page_rows * kRowBytes);
          }
          __syncwarp();                               // the expected bytes are set before any copy lands
          if (valid) {
            unsigned char* stage = smem + static_cast<size_t>(s) * kStageBytes;
            const uint32_t off = static_cast<uint32_t>(lane) * page_rows * 128u;
            tma_load_5d(stage + off, &kmap, 0, h, 0, cur, l, &full[s], policy);
            tma_load_5d(stage + kBoxBytes + off, &kmap, 64, h, 0, cur, l, &full[s], policy);
          }
        }
        if (more) {
          stash(buf ^ 1);
          cl = nl;
          ch = nh;
          cnp = nnp;
        }
        __syncwarp();                                 // the group's ids are read before they are replaced
      }
    } else if (warp == 0) {
      // ---------------- producer, packed layouts: one thread
      if (lane == 0) {
        Cursor c = cursor_at(g, t0);
        for (int t = t0; t < t1; ++t, ++k) {
          if (t > t0) cursor_next(g, c);
          const int row = packed_tile(g, c, a.scores).row;
#ifdef TRI_TEST_HOOKS
          if (t == g.test_skip_tile) continue;        // test builds: no copy and no arrival for this tile
#endif
          const int s = k % kStages, n = k / kStages;
          if (n > 0 && !*abort_flag && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) *abort_flag = 1;
          if (*abort_flag) continue;
          unsigned char* stage = smem + static_cast<size_t>(s) * kStageBytes;
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
          j_last = j;
        }
      } else {
        k += t1 - t0;
        j += t1 - t0;
      }
    } else {
      // ---------------- epilogue: one key per thread; warpgroup eg takes the
      // tiles of accumulator buffer eg (every kAccBufs-th tile of the walk)
      const int eg = (warp - 2) >> 2;
      const int quarter = warp & 3;                   // tensor-memory lanes 32*quarter ..
      const int r = quarter * 32 + lane;
      // Row r of a tile.  Whole-page PAGED tiles hold each page head-major:
      // page p = r >> (block_shift + head_shift), head (r >> block_shift) &
      // (H - 1), token p * block_size + (r & (block_size - 1)) of the tile;
      // a warp's 32 rows then hold min(H, 32 / block_size) heads (at least
      // one), consecutive from h_first.  Otherwise one head, row r = token r.
      const bool whole = a.whole_pages != 0;
      int tok = r, hr = 0, h_first = 0, heads_in_warp = 1;
      if (whole) {
        hr = (r >> g.block_shift) & (g.H - 1);
        tok = ((r >> (g.block_shift + a.head_shift)) << g.block_shift) | (r & (g.block_size - 1));
        h_first = ((quarter * 32) >> g.block_shift) & (g.H - 1);
        heads_in_warp = min(g.H, max(1, 32 >> g.block_shift));
      }
      // PAGED: the page id of this thread's key, loaded a tile of this
      // warpgroup ahead (the load's latency under a saturated memory system
      // is about a tile's time)
      const bool paged = g.layout == TRI_LAYOUT_PAGED;
      auto page_id = [&](const PagedTile& T) -> int32_t {
        return tok < T.tvalid ? g.block_table[T.tbl + (tok >> g.block_shift)] : -1;
      };
      // cc at tile t moves to tile t + kAccBufs (as far as the walk goes)
      auto step = [&](Cursor& cc, int t) {
        for (int i = 1; i <= kAccBufs && t + i < t1; ++i) cursor_next(g, cc);
      };
      const int j0 = j;
      const int first = t0 + (((eg - j0) % kAccBufs) + kAccBufs) % kAccBufs;
      j = j0 + (t1 - t0);                             // every epilogue warp's count after this run
      Cursor c{}, cn{};
      PagedTile Tn{};
      int32_t pg_n = -1;
      if (first < t1) {
        c = cursor_at(g, first);
        cn = c;
        step(cn, first);
        if (paged) {
          Tn = paged_tile(g, c, whole, a.scores);
          pg_n = page_id(Tn);
        }
      }
      for (int t = first; t < t1; t += kAccBufs) {
        if (t > first) {
          c = cn;
          step(cn, t);
        }
        const PagedTile Tc = Tn;
        const int32_t pg = pg_n;
        if (paged && t + kAccBufs < t1) {
          Tn = paged_tile(g, cn, whole, a.scores);
          pg_n = page_id(Tn);
        }
        const int jt = j0 + (t - t0);
        const int ab = jt % kAccBufs, na = jt / kAccBufs;
        // the tile's output, decoded while the MMAs run; keys in pages outside
        // the pool are not written
        float* out;
        bool live;
        if (paged) {
          out = Tc.out + hr * (static_cast<int64_t>(g.batch) * g.score_stride) + tok;
          live = tok < Tc.tvalid && static_cast<unsigned>(pg) < static_cast<unsigned>(g.num_blocks);
        } else {
          const PackedTile T = packed_tile(g, c, a.scores);
          out = T.out + tok;
          live = tok < T.rows;
        }
        if (!*abort_flag && !mbar_wait_bounded(&acc_full[ab], na & 1)) *abort_flag = 1;
        if (*abort_flag) continue;
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * kAccCols);
        // tcgen05.ld reads the same columns in every lane: the warp goes
        // through the columns of each head its rows hold, and each lane keeps
        // its own head's max
        float best = 0.f;
        for (int i = 0; i < heads_in_warp; ++i) {
          const int hh = h_first + i;
          float m = 0.f;
          // columns 2n, 2n + 1 = offset n's hi and lo products
          auto take = [&](const uint32_t* v, int cnt, int n0) {
#pragma unroll
            for (int e = 0; e < cnt / 2; ++e) {
              const float s2 = __uint_as_float(v[2 * e]) + __uint_as_float(v[2 * e + 1]);
              if (n0 + e < a.n_offsets) m = n0 + e == 0 ? s2 : fmaxf(m, s2);
            }
          };
          // up to two loads per wait; a load of 32 columns only from a
          // multiple of 32 (a head's block may start on an odd multiple of 16)
          const int c_head = hh * a.head_cols, c_end = c_head + a.head_cols;
          for (int col = c_head; col < c_end;) {
            const int w1 = ((col & 31) == 0 && c_end - col >= 32) ? 32 : 16;
            const int c2 = col + w1;
            const int w2 = c2 >= c_end ? 0 : ((c2 & 31) == 0 && c_end - c2 >= 32) ? 32 : 16;
            const uint32_t ca = taddr + static_cast<uint32_t>(col), cb = taddr + static_cast<uint32_t>(c2);
            const int n0 = (col - c_head) >> 1, n1 = (c2 - c_head) >> 1;
            if (w1 == 32 && w2 == 32) {
              uint32_t x[32], y[32];
              tmem_ld_pair(ca, cb, x, y);
              take(x, 32, n0);
              take(y, 32, n1);
            } else if (w1 == 32 && w2 == 16) {
              uint32_t x[32], y[16];
              tmem_ld_pair(ca, cb, x, y);
              take(x, 32, n0);
              take(y, 16, n1);
            } else if (w1 == 16 && w2 == 32) {
              uint32_t x[16], y[32];
              tmem_ld_pair(ca, cb, x, y);
              take(x, 16, n0);
              take(y, 32, n1);
            } else if (w2 != 0 || w1 == 32) {     // 16 + 16, or 32 as two 16s
              uint32_t x[16], y[16];
              tmem_ld_pair(ca, ca + 16u, x, y);
              take(x, 16, n0);
              take(y, 16, n0 + 8);
            } else {
              uint32_t x[16];
              tmem_ld_one(ca, x);
              take(x, 16, n0);
            }
            col += w1 + (w2 != 0 ? w2 : 0);
          }
          if (hh == hr) best = m;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        if (live) *out = best;
      }
    }
    t0 = t1;
    __syncthreads();   // the next run's weights overwrite B
  }

  // never exit with copies in flight, nor free tensor memory under MMAs still
  // running (only possible after an abort): the producer waits for its
  // copies, the MMA thread for its last commit (commits complete in order)
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int s = 0; s < kStages && s < k; ++s) mbar_wait_bounded(&full[s], ((k - 1 - s) / kStages) & 1);
  }
  if (warp == 1 && lane == 0 && *abort_flag && j_last >= 0)
    mbar_wait_bounded(&acc_full[j_last % kAccBufs], (j_last / kAccBufs) & 1);
  if (*abort_flag && threadIdx.x == 0) flag(TRI_DEVFLAG_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace smax
}  // namespace tri
