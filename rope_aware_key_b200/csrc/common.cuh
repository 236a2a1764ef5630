// Shared device-side pieces: cache geometry, row addressing, status word,
// mbarrier / bulk-copy PTX wrappers and block-level scans.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "tri_evict.h"

namespace tri {

constexpr int kD = TRI_HEAD_DIM;          // head_dim, elements
constexpr int kRowBytes = kD * 2;         // one bf16 row
constexpr int kRowVec = kRowBytes / 16;   // 16-byte vectors per row

// Everything a kernel needs to find a row of the cache.  Passed by value as
// a __grid_constant__ kernel parameter (about 3 KB).
struct Geom {
  int layout;                // tri_layout
  int L, H, batch;
  int block_size, max_blocks, num_blocks;
  int block_shift;           // PAGED: log2(block_size) when it is a power of two, else -1
  int v_host;                // V lives in pinned host memory mapped into the device (gather reads it over the bus)
  int pages_per_tile;        // PAGED: consecutive pages of a sequence scored as one tile
  int64_t sL, sH, sB;        // layer / head / (seq for CONTIG, page for PAGED) strides, elements
  int64_t score_stride;      // floats per score row
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* block_table;
  int32_t len[TRI_MAX_BATCH];         // keys per sequence
  int32_t start[TRI_MAX_BATCH];       // RAGGED: first token of the sequence
  int32_t tile_prefix[TRI_MAX_BATCH + 1];  // score tiles before sequence b (per layer-head or layer)
#ifdef TRI_TEST_HOOKS
  int test_skip_tile;        // test builds only: the score producer issues nothing for this tile (-1: none)
#endif
};

// Per-device status word; kernels OR TRI_DEVFLAG_* bits into it.
__device__ unsigned int g_status;

__device__ __forceinline__ void flag(unsigned int bits) { atomicOr(&g_status, bits); }

// Invariants of the selection and compaction (kept counts, histogram
// totals, holes against movers), checked on the device in a library built
// with -DTRI_CHECKED; a violation sets TRI_DEVFLAG_INVARIANT and the kernel
// carries on.  The product build compiles them out.
#ifdef TRI_CHECKED
#define TRI_CHECK(cond)                                   \
  do {                                                    \
    if (!(cond)) ::tri::flag(TRI_DEVFLAG_INVARIANT);      \
  } while (0)
#else
#define TRI_CHECK(cond) \
  do {                  \
  } while (0)
#endif

// Element offset of row i of unit (l, h, b).  For PAGED, *ok is cleared (and
// 0 returned) when the page id is outside the pool.
__device__ __forceinline__ int64_t row_elem(const Geom& g, int l, int h, int b, int i, bool* ok) {
  if (g.layout == TRI_LAYOUT_CONTIG)
    return l * g.sL + h * g.sH + b * g.sB + static_cast<int64_t>(i) * kD;
  if (g.layout == TRI_LAYOUT_RAGGED)
    return l * g.sL + h * g.sH + (static_cast<int64_t>(g.start[b]) + i) * kD;
  const int pg = g.block_shift >= 0 ? i >> g.block_shift : i / g.block_size;
  const int blk = g.block_table[static_cast<int64_t>(b) * g.max_blocks + pg];
  if (static_cast<unsigned>(blk) >= static_cast<unsigned>(g.num_blocks)) {
    *ok = false;
    return 0;
  }
  return l * g.sL + static_cast<int64_t>(blk) * g.sB +
         static_cast<int64_t>((i - pg * g.block_size) * g.H + h) * kD;
}

// Largest b in [0, batch) with prefix[b] <= r (prefix non-decreasing, prefix[0] = 0).
__device__ __forceinline__ int find_seq(const int32_t* prefix, int batch, int r) {
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= r) lo = mid;
    else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete, for at most about
// two seconds (a test build may set a shorter limit); on timeout set
// TRI_DEVFLAG_TIMEOUT and return false.
#ifndef TRI_WAIT_LIMIT_NS
#define TRI_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kWaitLimitNs = TRI_WAIT_LIMIT_NS;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      flag(TRI_DEVFLAG_TIMEOUT);
      return false;
    }
  }
}

// L2 policy for data read exactly once.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 1-D bulk copy global -> shared (no multicast), completing on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// 16-byte global load (plain: also right for pinned host memory mapped into
// the device's address space).
__device__ __forceinline__ uint4 ld_v4(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// 16-byte global load that bypasses L1 (read-only data).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ------------------------------------------------------------------ scans

// Exclusive block-wide sum of `v` for NT threads; *total gets the block sum.
// `sh` needs NT/32 words.  Contains __syncthreads(): call from all threads.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t v, uint32_t* sh, uint32_t* total) {
  static_assert(NT % 32 == 0 && NT <= 1024, "block size");
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = lane < NW ? sh[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) sh[lane] = s;
  }
  __syncthreads();
  uint32_t before = warp ? sh[warp - 1] : 0u;
  *total = sh[NW - 1];
  __syncthreads();
  return before + x - v;
}

}  // namespace tri
