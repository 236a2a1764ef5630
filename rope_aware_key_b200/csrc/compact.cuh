// Compaction of K and V to the kept keys (bit copies, 16 bytes per lane,
// a half-warp per 256-byte row).
//
// Page "The future-offset average in TriAttention can be precomputed",
// opening section: once the keys are scored, the cache keeps the highest
// within its budget and evicts the rest.  The pages do not say how the
// survivors are laid out; the two forms below are this library's reading
// (ascending order out of place; a hole fill that moves the fewest rows in
// place, which attention does not notice since K and V rows move together).
//
//  * gather (out of place): out[u][j] = cache row kept[u][j] of unit u, for
//    j < kept_count[u]; the output is [units][B][128] for K and for V.  A
//    warp copies a chunk of 32 consecutive kept rows of one unit.
//  * hole fill (in place): in a unit with n > B keys the kept keys below B
//    stay, and the evicted positions below B, ascending, receive the kept keys
//    at or above B, ascending.  Sources (>= B) and destinations (< B) are
//    disjoint, so one pass without any ordering between rows is race-free,
//    and only the rows that must move are touched.  Units that move few rows
//    take a warp each, which finds every mover's hole by a search over the
//    kept indices (no barrier); units that move many take a CTA each, which
//    lists the holes with a shared bitmap.
#pragma once

#include "common.cuh"

namespace tri {
namespace compact {

#ifndef TRI_GATHER_UNROLL
#define TRI_GATHER_UNROLL 2
#endif
#ifndef TRI_GATHER_BLOCKS_PER_SM
#define TRI_GATHER_BLOCKS_PER_SM 6
#endif

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = TRI_GATHER_UNROLL;     // rows in flight per half-warp
// The grid: this many CTAs per SM, walking the chunks grid-stride.  The kernel
// takes 57 registers, so 4 CTAs of 256 threads are resident per SM and the rest
// start as those finish; capping the registers so that all 6 are resident at
// once (40 registers), or launching only 4 per SM, measured slower (109.7 and
// 108.1 vs 103.0 us per gather on 288 x 2048 rows).
constexpr int kGatherBlocksPerSm = TRI_GATHER_BLOCKS_PER_SM;
constexpr int kChunkRows = 32;                      // kept rows of one unit per warp and step

__device__ __forceinline__ void unit_coords(const Geom& g, int u, int* l, int* h, int* b) {
  *b = u % g.batch;
  const int lh = u / g.batch;
  *l = lh / g.H;
  *h = lh - *l * g.H;
}

// A warp takes a chunk of kChunkRows consecutive kept rows of one unit: the
// unit, its base address and its kept indices (one coalesced load, then
// shuffles) are found once per chunk, and each half-warp copies rows with
// 2 x kGatherUnroll 16-byte loads in flight per lane before its stores.
__global__ void __launch_bounds__(kGatherThreads)
gather_kernel(const __grid_constant__ Geom g, const int32_t* __restrict__ kept,
              const int32_t* __restrict__ kept_count, int B, uint16_t* __restrict__ kout,
              uint16_t* __restrict__ vout, int chunks_per_unit, int total_chunks) {
  const int lane = threadIdx.x & 31;
  const int l16 = lane & 15, hw = lane >> 4;
  const int warp0 = (blockIdx.x * kGatherThreads + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * kGatherThreads) >> 5;
  const bool packed = g.layout != TRI_LAYOUT_PAGED;
  for (int c = warp0; c < total_chunks; c += nwarps) {
    const int u = c / chunks_per_unit;
    const int j0 = (c - u * chunks_per_unit) * kChunkRows;
    const int cnt = __ldg(kept_count + u);
#ifdef TRI_CHECKED
    if (j0 == 0 && lane == 0) {
      int l_, h_, b_;
      unit_coords(g, u, &l_, &h_, &b_);
      TRI_CHECK(cnt == min(B, g.len[b_]));         // the selection kept min(B, n)
    }
#endif
    const int rows = min(kChunkRows, cnt - j0);     // warp-uniform
    if (rows <= 0) continue;
    int l, h, b;
    unit_coords(g, u, &l, &h, &b);
    const int n = g.len[b];
    const int my_i = lane < rows ? __ldg(kept + static_cast<int64_t>(u) * B + j0 + lane) : 0;
    bool ok0 = true;
    const int64_t base = packed ? row_elem(g, l, h, b, 0, &ok0) : 0;
    const int64_t out0 = static_cast<int64_t>(u) * B + j0;
    for (int r0 = 0; r0 < rows; r0 += 2 * kGatherUnroll) {
      uint4 kx[kGatherUnroll], vx[kGatherUnroll];
      bool live[kGatherUnroll];
#pragma unroll
      for (int q = 0; q < kGatherUnroll; ++q) {
        const int r = r0 + 2 * q + hw;
        const int i = __shfl_sync(0xffffffffu, my_i, r & (kChunkRows - 1));
        live[q] = false;
        if (r >= rows) continue;
        if (static_cast<unsigned>(i) >= static_cast<unsigned>(n)) {
          if (l16 == 0) flag(TRI_DEVFLAG_BAD_KEPT);
          continue;
        }
        int64_t e = base + static_cast<int64_t>(i) * kD;
        if (!packed) {
          bool ok = true;
          e = row_elem(g, l, h, b, i, &ok);
          if (!ok) {
            if (l16 == 0) flag(TRI_DEVFLAG_BAD_PAGE);
            continue;
          }
        }
        kx[q] = ld_nc_v4(g.k + e + l16 * 8);
        vx[q] = g.v_host ? ld_v4(g.v + e + l16 * 8) : ld_nc_v4(g.v + e + l16 * 8);   // warp-uniform
        live[q] = true;
      }
#pragma unroll
      for (int q = 0; q < kGatherUnroll; ++q) {
        if (!live[q]) continue;
        const int64_t row = out0 + r0 + 2 * q + hw;
        reinterpret_cast<uint4*>(kout + row * kD)[l16] = kx[q];
        reinterpret_cast<uint4*>(vout + row * kD)[l16] = vx[q];
      }
    }
  }
}

// Hole fill, one warp per unit (units [blockIdx.x * kFillWarps, ...)), for
// units that move few rows (a row of B + a window of new tokens).  With
// the kept indices ascending, let f be the first kept index >= B: the m = B - f
// movers are kept[f .. B), and the r-th hole (the r-th position below B that
// is not kept) is at r + #{i < f : kept[i] - i <= r} -- z_i = kept[i] - i,
// the number of holes before kept[i], never decreases, so an upper bound
// search over it places every mover.  Each lane places one mover per step;
// then the movers' K and V rows are copied by half-warps (16 bytes a lane).
constexpr int kFillWarps = 4;
constexpr int kFillThreadsWarp = kFillWarps * 32;
constexpr int kFillWarpMovers = 512;               // rows moved per unit up to which a warp per unit is used

// The hole fill of one unit (n > B keys, kept ascending), by one warp.
__device__ __forceinline__ void holefill_unit_warp(const Geom& g, const int32_t* __restrict__ ku, int B, int n,
                                                   int l, int h, int b, uint16_t* k, uint16_t* v) {
  const int lane = threadIdx.x & 31, l16 = lane & 15, hw = lane >> 4;
  // f: the first kept index >= B (every lane searches the same range)
  int lo = 0, hi = B;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (ku[mid] >= B) hi = mid;
    else lo = mid + 1;
  }
  const int f = lo;
  const int m = B - f;                             // movers = holes below B
  // ascending kept indices: the last one below B sits just before the movers
  if (lane == 0) TRI_CHECK(f == 0 || ku[f - 1] < B);
  for (int r0 = 0; r0 < m; r0 += 32) {
    const int r = r0 + lane;
    int src = -1, dst = -1;
    if (r < m) {
      src = ku[f + r];
      // upper bound of r in z_i = kept[i] - i, i < f
      int a = 0, c = f;
      while (a < c) {
        const int mid = (a + c) >> 1;
        if (ku[mid] - mid <= r) a = mid + 1;
        else c = mid;
      }
      dst = r + a;
      if (src < B || src >= n || dst >= B) {       // not ascending, or out of the row
        flag(TRI_DEVFLAG_BAD_KEPT);
        src = -1;
      }
      if (r > 0) TRI_CHECK(ku[f + r - 1] < src || src < 0);    // movers ascending
    }
    const int cnt = min(32, m - r0);
    for (int q = 0; q < cnt; q += 2) {             // half-warp hw copies pair q + hw
      const int s_i = __shfl_sync(0xffffffffu, src, (q + hw) & 31);
      const int d_i = __shfl_sync(0xffffffffu, dst, (q + hw) & 31);
      if (q + hw >= cnt || s_i < 0) continue;
      bool ok = true;
      const int64_t es = row_elem(g, l, h, b, s_i, &ok);
      const int64_t ed = row_elem(g, l, h, b, d_i, &ok);
      if (!ok) {
        if (l16 == 0) flag(TRI_DEVFLAG_BAD_PAGE);
        continue;
      }
      const uint4 kx = ld_nc_v4(k + es + l16 * 8);
      const uint4 vx = ld_nc_v4(v + es + l16 * 8);
      reinterpret_cast<uint4*>(k + ed)[l16] = kx;
      reinterpret_cast<uint4*>(v + ed)[l16] = vx;
    }
  }
}

__global__ void __launch_bounds__(kFillThreadsWarp)
holefill_warp_kernel(const __grid_constant__ Geom g, const int32_t* __restrict__ kept, int B, uint16_t* k,
                     uint16_t* v, int units) {
  const int u = blockIdx.x * kFillWarps + (threadIdx.x >> 5);
  if (u >= units) return;                          // whole warps
  int l, h, b;
  unit_coords(g, u, &l, &h, &b);
  const int n = g.len[b];
  if (n <= B) return;
  holefill_unit_warp(g, kept + static_cast<int64_t>(u) * B, B, n, l, h, b, k, v);
}

// Hole fill, one CTA per unit, for units that move many rows (a long row
// pruned to B for the first time): a shared bitmap of the kept positions
// below B, the holes listed in order by a block scan, then 16 rows in flight
// per CTA.  Dynamic shared memory: ceil(B/32) + B words.
constexpr int kFillThreads = 256;
constexpr int kMaxFillCta = 16384;                 // largest B the CTA form's shared memory takes

__global__ void __launch_bounds__(kFillThreads)
holefill_cta_kernel(const __grid_constant__ Geom g, const int32_t* __restrict__ kept, int B, uint16_t* k,
                    uint16_t* v) {
  extern __shared__ uint32_t fill_smem[];
  __shared__ uint32_t scan_sh[kFillThreads / 32];
  const int u = blockIdx.x;
  int l, h, b;
  unit_coords(g, u, &l, &h, &b);
  const int n = g.len[b];
  if (n <= B) return;
  const int32_t* __restrict__ ku = kept + static_cast<int64_t>(u) * B;
  const int words = (B + 31) >> 5;
  uint32_t* bitmap = fill_smem;
  int32_t* holes = reinterpret_cast<int32_t*>(fill_smem + words);

  for (int w = threadIdx.x; w < words; w += kFillThreads) bitmap[w] = 0u;
  __syncthreads();
  for (int j = threadIdx.x; j < B; j += kFillThreads) {
    const int i = ku[j];
    if (i >= 0 && i < B) atomicOr(&bitmap[i >> 5], 1u << (i & 31));
  }
  __syncthreads();

  // holes in ascending order
  uint32_t base = 0;
  for (int w0 = 0; w0 < words; w0 += kFillThreads) {
    const int w = w0 + threadIdx.x;
    uint32_t m = 0u;
    if (w < words) {
      const uint32_t valid = (w == words - 1 && (B & 31)) ? ((1u << (B & 31)) - 1u) : 0xffffffffu;
      m = ~bitmap[w] & valid;
    }
    uint32_t total;
    uint32_t pos = base + block_exclusive_sum<kFillThreads>(__popc(m), scan_sh, &total);
    while (m) {
      const int bit = __ffs(m) - 1;
      holes[pos++] = w * 32 + bit;
      m &= m - 1u;
    }
    base += total;
  }
  __syncthreads();

  const int nh = static_cast<int>(base);
  const int first_mover = B - nh;                  // kept[first_mover..B) are >= B
  if (threadIdx.x == 0) TRI_CHECK(first_mover == 0 || ku[first_mover - 1] < B);
  const int l16 = threadIdx.x & 15;
  for (int r = threadIdx.x >> 4; r < nh; r += kFillThreads / 16) {
    const int src_i = ku[first_mover + r];
    const int dst_i = holes[r];
    if (src_i < B || src_i >= n) {
      if (l16 == 0) flag(TRI_DEVFLAG_BAD_KEPT);
      continue;
    }
    if (l16 == 0 && r > 0) TRI_CHECK(ku[first_mover + r - 1] < src_i);    // movers ascending
    bool ok = true;
    const int64_t es = row_elem(g, l, h, b, src_i, &ok);
    const int64_t ed = row_elem(g, l, h, b, dst_i, &ok);
    if (!ok) {
      if (l16 == 0) flag(TRI_DEVFLAG_BAD_PAGE);
      continue;
    }
    const uint4 kx = ld_nc_v4(k + es + l16 * 8);
    const uint4 vx = ld_nc_v4(v + es + l16 * 8);
    reinterpret_cast<uint4*>(k + ed)[l16] = kx;
    reinterpret_cast<uint4*>(v + ed)[l16] = vx;
  }
}

}  // namespace compact
}  // namespace tri
