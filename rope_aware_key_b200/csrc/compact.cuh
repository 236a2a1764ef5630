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
//    j < kept_count[u]; the output is [units][B][128] for K and for V.
//  * hole fill (in place): in a unit with n > B keys the kept keys below B
//    stay, and the evicted positions below B, ascending, receive the kept keys
//    at or above B, ascending.  Sources (>= B) and destinations (< B) are
//    disjoint, so one pass without any ordering between rows is race-free,
//    and only the rows that must move are touched.
#pragma once

#include "common.cuh"

namespace tri {
namespace compact {

#ifndef TRI_GATHER_ROWS
#define TRI_GATHER_ROWS 2
#endif
#ifndef TRI_GATHER_BLOCKS_PER_SM
#define TRI_GATHER_BLOCKS_PER_SM 16
#endif

constexpr int kGatherThreads = 256;
constexpr int kGatherRows = TRI_GATHER_ROWS;
constexpr int kGatherBlocksPerSm = TRI_GATHER_BLOCKS_PER_SM;
constexpr int kFillThreads = 256;
constexpr int kMaxFillBudget = 16384;

__device__ __forceinline__ void unit_coords(const Geom& g, int u, int* l, int* h, int* b) {
  *b = u % g.batch;
  const int lh = u / g.batch;
  *l = lh / g.H;
  *h = lh - *l * g.H;
}

// Each half-warp copies kGatherRows rows per step (all loads issued before
// the stores, so 2 x kGatherRows x 16 bytes per lane are in flight).
__global__ void __launch_bounds__(kGatherThreads)
gather_kernel(const __grid_constant__ Geom g, const int32_t* __restrict__ kept,
              const int32_t* __restrict__ kept_count, int B, uint16_t* __restrict__ kout,
              uint16_t* __restrict__ vout, int total_rows) {
  // total_rows = units * B < 2^31 (checked on the host)
  const int l16 = threadIdx.x & 15;
  const int hw = (blockIdx.x * kGatherThreads + threadIdx.x) >> 4;
  const int nhw = (gridDim.x * kGatherThreads) >> 4;
  for (int base = hw; base < total_rows; base += nhw * kGatherRows) {
    uint4 kx[kGatherRows], vx[kGatherRows];
    bool live[kGatherRows];
#pragma unroll
    for (int r = 0; r < kGatherRows; ++r) {
      const int row = base + r * nhw;
      live[r] = false;
      if (row >= total_rows) continue;
      const int u = row / B;
      const int j = row - u * B;
      if (j >= __ldg(kept_count + u)) continue;
      const int i = __ldg(kept + row);
      int l, h, b;
      unit_coords(g, u, &l, &h, &b);
      if (static_cast<unsigned>(i) >= static_cast<unsigned>(g.len[b])) {
        if (l16 == 0) flag(TRI_DEVFLAG_BAD_KEPT);
        continue;
      }
      bool ok = true;
      const int64_t e = row_elem(g, l, h, b, i, &ok);
      if (!ok) {
        if (l16 == 0) flag(TRI_DEVFLAG_BAD_PAGE);
        continue;
      }
      kx[r] = ld_nc_v4(g.k + e + l16 * 8);
      vx[r] = ld_nc_v4(g.v + e + l16 * 8);
      live[r] = true;
    }
#pragma unroll
    for (int r = 0; r < kGatherRows; ++r) {
      if (!live[r]) continue;
      const int64_t row = base + r * nhw;
      reinterpret_cast<uint4*>(kout + row * kD)[l16] = kx[r];
      reinterpret_cast<uint4*>(vout + row * kD)[l16] = vx[r];
    }
  }
}

// One CTA per unit.  Dynamic shared memory: bitmap of the kept positions
// below B (ceil(B/32) words) followed by the list of holes (B ints).
__global__ void __launch_bounds__(kFillThreads)
holefill_kernel(const __grid_constant__ Geom g, const int32_t* __restrict__ kept, int B,
                uint16_t* k, uint16_t* v) {
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
  const int first_mover = B - nh;         // kept[first_mover..B) are >= B
  const int l16 = threadIdx.x & 15;
  for (int r = threadIdx.x >> 4; r < nh; r += kFillThreads / 16) {
    const int src_i = ku[first_mover + r];
    const int dst_i = holes[r];
    if (src_i < B || src_i >= n) {
      if (l16 == 0) flag(TRI_DEVFLAG_BAD_KEPT);
      continue;
    }
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
