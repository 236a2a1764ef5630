// C ABI of the library (declared in include/tri_evict.h): argument checks on
// the host, geometry packing, and the kernel launches.  Everything runs on
// the caller's stream; nothing is allocated, freed or synchronised here
// (tri_read_device_status excepted, which waits for its own small copy).
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tri_evict.h"
#include "common.cuh"
#include "fold.cuh"
#include "score.cuh"
#include "select.cuh"
#include "select_warp.cuh"
#include "compact.cuh"
#include "score_max.cuh"
#include "score_pos.cuh"
#include "score_pos_tma.cuh"
#include "fused.cuh"

namespace {

using tri::Geom;

std::atomic<uint64_t> g_launches{0};
thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int score_blocks_per_sm = 0;
  int smax_blocks_per_sm = 0;
  int pos_blocks_per_sm = 0;
  int pt_blocks_per_sm = 0;
  int fused_cluster = 0;        // cluster size of the single-kernel step (0: unavailable)
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

tri_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return TRI_ERR_CUDA;
}

#define TRI_CUDA(call)                               \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_fail(e_);     \
  } while (0)

// The driver's current-context calls, looked up once through the runtime
// (the library links the runtime statically and does not link libcuda).
struct CtxCalls {
  PFN_cuCtxGetCurrent_v4000 get = nullptr;
  PFN_cuCtxSetCurrent_v4000 set = nullptr;
};
const CtxCalls& ctx_calls() {
  static CtxCalls c;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      c.get = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxSetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      c.set = reinterpret_cast<PFN_cuCtxSetCurrent_v4000>(p);
  });
  return c;
}

// The device a call works on is made current for the length of the call
// only: the runtime's current device belongs to the caller's host thread,
// so the caller's own context (possibly none) is put back when the scope
// ends.  Nothing is switched when the caller is already on that device.
class DeviceScope {
 public:
  DeviceScope() = default;
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;
  ~DeviceScope() {
    if (!switched_) return;
    const CtxCalls& c = ctx_calls();
    if (c.set) c.set(saved_ctx_);
    else if (saved_dev_ >= 0) cudaSetDevice(saved_dev_);
  }
  // Make `dev` current (remembering what was current before).
  cudaError_t enter(int dev) {
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return e;
    if (cur == dev) return cudaSuccess;
    const CtxCalls& c = ctx_calls();
    saved_ctx_ = nullptr;
    if (c.get) c.get(&saved_ctx_);
    saved_dev_ = cur;
    e = cudaSetDevice(dev);
    if (e == cudaSuccess) switched_ = true;
    return e;
  }

 private:
  bool switched_ = false;
  CUcontext saved_ctx_ = nullptr;
  int saved_dev_ = -1;
};

// Make the device that owns `ptr` current for the scope's lifetime, and set
// up per-device state once.
tri_status use_device_of(const void* ptr, int* dev_out, DeviceScope* scope) {
  int dev = -1;
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, ptr);
  if (e != cudaSuccess) return cuda_fail(e);
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return TRI_ERR_INVALID_ARG;
  dev = attr.device;
  if (dev < 0 || dev >= kMaxDevices) return TRI_ERR_UNSUPPORTED;
  TRI_CUDA(scope->enter(dev));
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    TRI_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    TRI_CUDA(cudaFuncSetAttribute(tri::score::score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::score::kSmemBytes)));
    TRI_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.score_blocks_per_sm, tri::score::score_kernel,
                                                           tri::score::kThreads, tri::score::kSmemBytes));
    if (d.score_blocks_per_sm < 1) return TRI_ERR_UNSUPPORTED;
    int pos_occ[2];
    TRI_CUDA(cudaFuncSetAttribute(tri::score::score_pos_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::score::kPosSmemBytes)));
    TRI_CUDA(cudaFuncSetAttribute(tri::score::score_pos_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::score::kPosSmemBytes)));
    TRI_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&pos_occ[0], tri::score::score_pos_kernel<0>,
                                                           tri::score::kThreads, tri::score::kPosSmemBytes));
    TRI_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&pos_occ[1], tri::score::score_pos_kernel<1>,
                                                           tri::score::kThreads, tri::score::kPosSmemBytes));
    d.pos_blocks_per_sm = pos_occ[0] < pos_occ[1] ? pos_occ[0] : pos_occ[1];
    if (d.pos_blocks_per_sm < 1) return TRI_ERR_UNSUPPORTED;
    TRI_CUDA(cudaFuncSetAttribute(tri::score::score_pos_tma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::score::kPtSmemBytes)));
    TRI_CUDA(cudaFuncSetAttribute(tri::score::score_pos_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::score::kPtSmemBytes)));
    TRI_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&pos_occ[0], tri::score::score_pos_tma_kernel<0>,
                                                           tri::score::kPtThreads, tri::score::kPtSmemBytes));
    TRI_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&pos_occ[1], tri::score::score_pos_tma_kernel<1>,
                                                           tri::score::kPtThreads, tri::score::kPtSmemBytes));
    d.pt_blocks_per_sm = pos_occ[0] < pos_occ[1] ? pos_occ[0] : pos_occ[1];
    if (d.pt_blocks_per_sm < 1) return TRI_ERR_UNSUPPORTED;
    TRI_CUDA(cudaFuncSetAttribute(tri::select::select_kernel<512>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  tri::select::kMaxShared));
    TRI_CUDA(cudaFuncSetAttribute(tri::select::select_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  tri::select::kMaxShared));
    TRI_CUDA(cudaFuncSetAttribute(tri::compact::holefill_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ((tri::compact::kMaxFillCta + 31) / 32 + tri::compact::kMaxFillCta) * 4));
    TRI_CUDA(cudaFuncSetAttribute(tri::select::select_warp_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::select::kWarpSmemBytes)));
    TRI_CUDA(cudaFuncSetAttribute(tri::select::select_warp_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::select::kWarpSmemBytes)));
    TRI_CUDA(cudaFuncSetAttribute(tri::smax::score_max_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::smax::kSmemBytes)));
    TRI_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.smax_blocks_per_sm, tri::smax::score_max_kernel,
                                                           tri::smax::kThreads, tri::smax::kSmemBytes));
    if (d.smax_blocks_per_sm < 1) return TRI_ERR_UNSUPPORTED;
    // the single-kernel step: clusters of 16 CTAs if the device can hold one, else 8
    TRI_CUDA(cudaFuncSetAttribute(tri::fused::fused_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::fused::kSmemBytes)));
    TRI_CUDA(cudaFuncSetAttribute(tri::fused::fused_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    TRI_CUDA(cudaFuncSetAttribute(tri::fused::fused_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(tri::fused::kSmemBytes)));
    for (int cs : {16, 8}) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = cs;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.gridDim = dim3(cs);
      cfg.blockDim = dim3(tri::fused::kThreads);
      cfg.dynamicSmemBytes = tri::fused::kSmemBytes;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      const cudaError_t e = cs == 16
          ? cudaOccupancyMaxActiveClusters(&clusters, tri::fused::fused_kernel<16>, &cfg)
          : cudaOccupancyMaxActiveClusters(&clusters, tri::fused::fused_kernel<8>, &cfg);
      if (e == cudaSuccess && clusters > 0) {
        d.fused_cluster = cs;
        break;
      }
      (void)cudaGetLastError();
    }
    d.ready = true;
  }
  *dev_out = dev;
  return TRI_OK;
}

// Where V lives, for a compaction on device `dev`: device memory of that
// device, or -- for OUT_OF_PLACE only, where V is read and never written --
// pinned host memory mapped into the device's address space at the same
// address (the gather then reads just the kept rows over the bus).  Sets
// g->v_host.
tri_status check_values(const tri_cache_desc* desc, int dev, tri_compact_mode mode, Geom* g) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, desc->v);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return TRI_ERR_INVALID_ARG;
  }
  if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
    if (attr.device != dev) return TRI_ERR_INVALID_ARG;
    g->v_host = 0;
    return TRI_OK;
  }
  if (attr.type == cudaMemoryTypeHost && attr.devicePointer == desc->v && mode == TRI_COMPACT_OUT_OF_PLACE) {
    g->v_host = 1;
    return TRI_OK;
  }
  return TRI_ERR_INVALID_ARG;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Score matrix of tri_compress_noalloc: a fixed array in the module's device
// memory (every device that loads the library holds it until exit), shared
// by all calls.  Host code may not use the symbol as a device address; its
// address is looked up once per device with that device current.
static __device__ __align__(256) float g_noalloc_scores[TRI_NOALLOC_MAX_SCORES];
float* g_noalloc_ptr[kMaxDevices] = {};

// Validate `c` and fill `g` (everything except the per-call pointers the
// kernels take separately).  `need_v`: compaction needs V.
tri_status make_geom(const tri_cache_desc* c, bool need_v, Geom* g) {
  if (!c || !g) return TRI_ERR_INVALID_ARG;
  if (c->head_dim != TRI_HEAD_DIM) return TRI_ERR_UNSUPPORTED;
  if (c->num_layers < 1 || c->num_kv_heads < 1 || c->batch < 1) return TRI_ERR_INVALID_ARG;
  if (c->batch > TRI_MAX_BATCH) return TRI_ERR_UNSUPPORTED;
  if (!c->k || !aligned16(c->k)) return TRI_ERR_INVALID_ARG;
  if (need_v && (!c->v || !aligned16(c->v))) return TRI_ERR_INVALID_ARG;
  if (c->v && !aligned16(c->v)) return TRI_ERR_INVALID_ARG;
  const int64_t L = c->num_layers, H = c->num_kv_heads, Bt = c->batch;
  if ((L * H * Bt) > (int64_t{1} << 31) - 1) return TRI_ERR_UNSUPPORTED;
  if (c->stride_layer < 0 || (c->stride_layer % 8) != 0) return TRI_ERR_INVALID_ARG;
  if (L > 1 && c->stride_layer == 0) return TRI_ERR_INVALID_ARG;

  std::memset(g, 0, sizeof(*g));
  g->layout = c->layout;
  g->L = c->num_layers;
  g->H = c->num_kv_heads;
  g->batch = c->batch;
  g->sL = c->stride_layer;
  g->k = static_cast<const uint16_t*>(c->k);
  g->v = static_cast<const uint16_t*>(c->v);

  int64_t max_len = 0;
  switch (c->layout) {
    case TRI_LAYOUT_CONTIG: {
      if (c->seq_len < 0) return TRI_ERR_INVALID_ARG;
      if (c->stride_head < 0 || c->stride_seq < 0 || (c->stride_head % 8) || (c->stride_seq % 8))
        return TRI_ERR_INVALID_ARG;
      if ((H > 1 && c->stride_head == 0) || (Bt > 1 && c->stride_seq == 0)) return TRI_ERR_INVALID_ARG;
      for (int b = 0; b < c->batch; ++b) g->len[b] = c->seq_len;
      g->sH = c->stride_head;
      g->sB = c->stride_seq;
      max_len = c->seq_len;
      break;
    }
    case TRI_LAYOUT_RAGGED: {
      if (!c->cu_seqlens) return TRI_ERR_INVALID_ARG;
      if (c->cu_seqlens[0] != 0) return TRI_ERR_INVALID_ARG;
      if (c->stride_head < 0 || (c->stride_head % 8)) return TRI_ERR_INVALID_ARG;
      if (H > 1 && c->stride_head == 0) return TRI_ERR_INVALID_ARG;
      for (int b = 0; b < c->batch; ++b) {
        // in 64 bits: the int32 difference of hostile offsets could wrap
        const int64_t n = int64_t{c->cu_seqlens[b + 1]} - c->cu_seqlens[b];
        if (n < 0 || n > INT32_MAX) return TRI_ERR_INVALID_ARG;
        g->len[b] = static_cast<int32_t>(n);
        g->start[b] = c->cu_seqlens[b];
        if (n > max_len) max_len = n;
      }
      g->sH = c->stride_head;
      break;
    }
    case TRI_LAYOUT_PAGED: {
      if (!c->seq_lens || !c->block_table) return TRI_ERR_INVALID_ARG;
      if (c->block_size < 1 || c->max_blocks_per_seq < 1 || c->num_blocks < 1) return TRI_ERR_INVALID_ARG;
      if (8 % c->num_kv_heads != 0 || int64_t{c->block_size} * c->num_kv_heads > tri::score::kTileRows)
        return TRI_ERR_UNSUPPORTED;
      const int64_t page = int64_t{c->block_size} * c->num_kv_heads * TRI_HEAD_DIM;
      if (c->stride_block < page || (c->stride_block % 8)) return TRI_ERR_INVALID_ARG;
      for (int b = 0; b < c->batch; ++b) {
        const int32_t n = c->seq_lens[b];
        if (n < 0 || int64_t{n} > int64_t{c->max_blocks_per_seq} * c->block_size) return TRI_ERR_INVALID_ARG;
        g->len[b] = n;
        if (n > max_len) max_len = n;
      }
      g->block_size = c->block_size;
      g->block_shift = (c->block_size & (c->block_size - 1)) == 0 ? __builtin_ctz(c->block_size) : -1;
      // as many consecutive pages per score tile as fill its 128 rows (at most 32)
      g->pages_per_tile = static_cast<int>(std::min<int64_t>(32, tri::score::kTileRows / (int64_t{c->block_size} * H)));
      g->max_blocks = c->max_blocks_per_seq;
      g->num_blocks = c->num_blocks;
      g->sB = c->stride_block;
      g->block_table = c->block_table;
      if (reinterpret_cast<uintptr_t>(c->block_table) & 3u) return TRI_ERR_INVALID_ARG;
      break;
    }
    default:
      return TRI_ERR_INVALID_ARG;
  }
  if (c->max_seq_len < 0) return TRI_ERR_INVALID_ARG;
  if (c->max_seq_len > 0 && c->max_seq_len < max_len) return TRI_ERR_INVALID_ARG;
  const int64_t cap = c->max_seq_len > 0 ? c->max_seq_len : max_len;
  if (cap > (int64_t{1} << 30)) return TRI_ERR_UNSUPPORTED;
  g->score_stride = (cap + 3) & ~int64_t{3};
  return TRI_OK;
}

// Score tiles: per sequence, 128-key chunks (CONTIG / RAGGED) or groups of
// pages_per_tile pages (PAGED).
// Returns the tile count, or INT64_MAX when the per-sequence prefix would not
// fit the int32 table the kernels search (callers reject counts > INT32_MAX).
int64_t fill_tile_prefix(Geom* g) {
  int64_t acc = 0;
  for (int b = 0; b < g->batch; ++b) {
    g->tile_prefix[b] = static_cast<int32_t>(acc);
    const int64_t per = g->layout == TRI_LAYOUT_PAGED ? int64_t{g->block_size} * g->pages_per_tile
                                                      : int64_t{tri::score::kTileRows};
    acc += (g->len[b] + per - 1) / per;
    if (acc > INT32_MAX) return INT64_MAX;
  }
  g->tile_prefix[g->batch] = static_cast<int32_t>(acc);
  const int64_t outer = g->layout == TRI_LAYOUT_PAGED ? g->L : int64_t{g->L} * g->H;
  return outer * acc;                                  // < 2^31 * 2^31
}

#ifdef TRI_TEST_HOOKS
// Test builds only: the score tile whose copy the producer leaves out (-1: none).
std::atomic<int> g_test_skip_tile{-1};
#endif

tri_status launch_score(const Geom& g0, const float* w, float* scores, int dev, cudaStream_t s) {
  Geom g = g0;
#ifdef TRI_TEST_HOOKS
  g.test_skip_tile = g_test_skip_tile.load();
#endif
  const int64_t ntiles = fill_tile_prefix(&g);
  if (ntiles == 0) return TRI_OK;
  if (ntiles > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  const int64_t resident = int64_t{g_dev[dev].sms} * g_dev[dev].score_blocks_per_sm;
  const int grid = static_cast<int>(ntiles < resident ? ntiles : resident);
  tri::score::score_kernel<<<grid, tri::score::kThreads, tri::score::kSmemBytes, s>>>(
      g, w, scores, static_cast<int>(ntiles));
  ++g_launches;
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

// Keys in the longest row.
int max_row(const Geom& g) {
  int max_len = 0;
  for (int b = 0; b < g.batch; ++b) max_len = g.len[b] > max_len ? g.len[b] : max_len;
  return max_len;
}

// How one selection launch is shaped, decided (and checked) on the host
// before anything is launched: a warp per row when every row holds at most
// kWarpMaxRow keys, else a CTA per row with its working set in shared memory.
struct SelectPlan {
  bool warp = false;     // the warp kernel (rows of at most kWarpMaxRow keys)
  int cap = 0, lcap = 0;
  size_t smem = 0;
};

tri_status plan_select(const Geom& g, int B, SelectPlan* p) {
  const int max_len = max_row(g);
  *p = SelectPlan();
  if (max_len <= tri::select::kWarpMaxRow) {
    p->warp = true;
    p->smem = tri::select::kWarpSmemBytes;
    return TRI_OK;
  }
  p->cap = (max_len + 3) & ~3;
  p->lcap = tri::select::list_capacity(B, p->cap);
  p->smem = tri::select::smem_bytes(p->cap, p->lcap);
  if (p->smem > static_cast<size_t>(tri::select::kMaxShared)) return TRI_ERR_UNSUPPORTED;
  return TRI_OK;
}

// fill: the in-place hole fill runs in the warp selection kernel, row by row
// (only with p.warp; see fill_in_select).
tri_status launch_select(const Geom& g, const SelectPlan& p, const float* scores, int B, int32_t* kept,
                         int32_t* kept_count, cudaStream_t s, bool fill = false) {
  const int units = g.L * g.H * g.batch;
  tri::select::Args a{scores, kept, kept_count, B, p.cap, p.lcap};
  if (p.warp) {
    const int grid = (units + tri::select::kWarpRows - 1) / tri::select::kWarpRows;
    uint16_t* k = const_cast<uint16_t*>(g.k);
    uint16_t* v = const_cast<uint16_t*>(g.v);
    if (fill)
      tri::select::select_warp_kernel<true><<<grid, tri::select::kWarpThreads, p.smem, s>>>(g, a, units, k, v);
    else
      tri::select::select_warp_kernel<false><<<grid, tri::select::kWarpThreads, p.smem, s>>>(g, a, units, k, v);
  } else if (p.cap >= 8192) {
    tri::select::select_kernel<512><<<units, 512, p.smem, s>>>(g, a);
  } else {
    tri::select::select_kernel<256><<<units, 256, p.smem, s>>>(g, a);
  }
  ++g_launches;
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

// Host checks of a compaction launch (everything launch_compact would refuse).
tri_status check_compact_launch(const Geom& g, int B, tri_compact_mode mode) {
  if (mode == TRI_COMPACT_OUT_OF_PLACE && int64_t{g.L} * g.H * g.batch * B > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  return TRI_OK;
}

// In-place compaction whose rows move few keys (at most kFillWarpMovers, the
// bound the standalone kernels also use for a warp per unit): a warp per row
// selects and then fills the row's holes in one kernel.
bool fill_in_select(const Geom& g, const SelectPlan& p, int B, tri_compact_mode mode) {
  return mode == TRI_COMPACT_IN_PLACE_HOLEFILL && p.warp && max_row(g) - B <= tri::compact::kFillWarpMovers;
}

tri_status launch_compact(const Geom& g, const int32_t* kept, const int32_t* kept_count, int B,
                          tri_compact_mode mode, void* k_out, void* v_out, int dev, cudaStream_t s) {
  const int units = g.L * g.H * g.batch;
  if (check_compact_launch(g, B, mode) != TRI_OK) return TRI_ERR_UNSUPPORTED;
  if (mode == TRI_COMPACT_OUT_OF_PLACE) {
    const int chunks_per_unit = (B + tri::compact::kChunkRows - 1) / tri::compact::kChunkRows;
    const int64_t chunks = int64_t{units} * chunks_per_unit;          // <= units * B <= INT32_MAX
    constexpr int kWarps = tri::compact::kGatherThreads / 32;
    const int64_t want = (chunks + kWarps - 1) / kWarps;
    const int64_t cap = int64_t{g_dev[dev].sms} * tri::compact::kGatherBlocksPerSm;
    const int grid = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
    tri::compact::gather_kernel<<<grid, tri::compact::kGatherThreads, 0, s>>>(
        g, kept, kept_count, B, static_cast<uint16_t*>(k_out), static_cast<uint16_t*>(v_out), chunks_per_unit,
        static_cast<int>(chunks));
  } else {
    // rows moved per unit: at most n - B; a warp per unit while that is small
    if (max_row(g) - B <= tri::compact::kFillWarpMovers || B > tri::compact::kMaxFillCta) {
      const int grid = (units + tri::compact::kFillWarps - 1) / tri::compact::kFillWarps;
      tri::compact::holefill_warp_kernel<<<grid, tri::compact::kFillThreadsWarp, 0, s>>>(
          g, kept, B, const_cast<uint16_t*>(g.k), const_cast<uint16_t*>(g.v), units);
    } else {
      const size_t smem = static_cast<size_t>((B + 31) / 32 + B) * 4;
      tri::compact::holefill_cta_kernel<<<units, tri::compact::kFillThreads, smem, s>>>(
          g, kept, B, const_cast<uint16_t*>(g.k), const_cast<uint16_t*>(g.v));
    }
  }
  ++g_launches;
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

// The single-kernel step (fused.cuh), when it applies: out-of-place
// compaction of a CONTIG or RAGGED cache whose units fill at most one wave of
// clusters and whose longest row fits the cluster's slices.  Returns
// TRI_ERR_UNSUPPORTED when it does not apply (the caller then runs the three
// kernels).
tri_status launch_fused(const Geom& g, const float* w, float* scores, int B, int32_t* kept, int32_t* kept_count,
                        void* k_out, void* v_out, int dev, cudaStream_t s) {
  const int C = g_dev[dev].fused_cluster;
  if (C == 0 || g.layout == TRI_LAYOUT_PAGED) return TRI_ERR_UNSUPPORTED;
  const int64_t units = int64_t{g.L} * g.H * g.batch;
  if (units * C > g_dev[dev].sms) return TRI_ERR_UNSUPPORTED;
  const int max_len = max_row(g);
  // Longer rows stream faster through the standalone scorer on every SM than
  // through one cluster per unit (measured: 1 x 4096 keys 20 vs 25 us per
  // step, 8 x 8192 even, 1 x 32768 33 vs 25 us).
  if (max_len > tri::fused::kMaxRow) return TRI_ERR_UNSUPPORTED;
  const int per = ((max_len + C - 1) / C + tri::score::kTileRows - 1) / tri::score::kTileRows * tri::score::kTileRows;
  if (per > tri::fused::kMaxSlice) return TRI_ERR_UNSUPPORTED;
  tri::fused::Args a{w, scores, kept, kept_count, static_cast<uint16_t*>(k_out), static_cast<uint16_t*>(v_out), B,
                     per > 0 ? per : tri::score::kTileRows};
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = C;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(units * C));
  cfg.blockDim = dim3(tri::fused::kThreads);
  cfg.dynamicSmemBytes = tri::fused::kSmemBytes;
  cfg.stream = s;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  const cudaError_t e = C == 16 ? cudaLaunchKernelEx(&cfg, tri::fused::fused_kernel<16>, g, a)
                                : cudaLaunchKernelEx(&cfg, tri::fused::fused_kernel<8>, g, a);
  ++g_launches;
  if (e != cudaSuccess) return cuda_fail(e);
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

tri_status check_compact_args(const tri_cache_desc* desc, const int32_t* kept, const int32_t* kept_count,
                              int B, tri_compact_mode mode, void* k_out, void* v_out) {
  if (!kept || !kept_count || B < 1) return TRI_ERR_INVALID_ARG;
  if (mode == TRI_COMPACT_OUT_OF_PLACE) {
    if (!k_out || !v_out || !aligned16(k_out) || !aligned16(v_out)) return TRI_ERR_INVALID_ARG;
  } else if (mode == TRI_COMPACT_IN_PLACE_HOLEFILL) {
    if (k_out || v_out) return TRI_ERR_INVALID_ARG;
  } else {
    return TRI_ERR_INVALID_ARG;
  }
  (void)desc;
  return TRI_OK;
}


// Everything the three stages of a compress call would refuse, checked on
// the host before the first launch (so an error return has launched nothing).
tri_status compress_checks(const Geom& g0, int B, tri_compact_mode mode, SelectPlan* plan) {
  Geom g = g0;
  if (fill_tile_prefix(&g) > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  tri_status st = plan_select(g0, B, plan);
  if (st != TRI_OK) return st;
  return check_compact_launch(g0, B, mode);
}

// The stages of tri_compress / tri_compress_noalloc once their checks have
// passed: the single-kernel step where it applies, else score, select,
// compact (in place with rows that move few keys: score, then the selection
// with the hole fill in it).
tri_status run_compress(const Geom& g, const SelectPlan& plan, const float* w, int B, tri_compact_mode mode,
                        int32_t* kept, int32_t* kept_count, void* k_out, void* v_out, float* scores, int dev,
                        cudaStream_t s) {
  tri_status st;
  if (mode == TRI_COMPACT_OUT_OF_PLACE) {
    st = launch_fused(g, w, scores, B, kept, kept_count, k_out, v_out, dev, s);
    if (st != TRI_ERR_UNSUPPORTED) return st;
  }
  st = launch_score(g, w, scores, dev, s);
  if (st != TRI_OK) return st;
  const bool fill = fill_in_select(g, plan, B, mode);
  st = launch_select(g, plan, scores, B, kept, kept_count, s, fill);
  if (st != TRI_OK || fill) return st;
  return launch_compact(g, kept, kept_count, B, mode, k_out, v_out, dev, s);
}

// The averaged fold: A_f = (1/|D|) sum_delta e^{i w_f delta} * e^{i w_f delta0}
// summed here in fp64 (in schedule order), then one launch maps the centers.
// The factors of the last schedule are kept (the caller holds the fold lock):
// a schedule rarely changes between calls, and |D| x 64 host sines and
// cosines cost more than the launch for long schedules.
struct FoldCache {
  bool valid = false;
  double theta = 0.0, delta0 = 0.0;
  std::vector<double> offsets;
  double a_re[tri::fold::kBands], a_im[tri::fold::kBands];
};

void launch_fold_mean(const tri_fold_params* p, const float* q_center, int n_centers, float* w_out, cudaStream_t s) {
  static FoldCache cache;
  tri::fold::FoldArgs a;
  a.q = q_center;
  a.w = w_out;
  a.n_centers = n_centers;
  a.pairing = p->pairing;
  const bool same = cache.valid && cache.theta == p->theta && cache.delta0 == p->delta0 &&
                    cache.offsets.size() == static_cast<size_t>(p->n_offsets) &&
                    std::equal(cache.offsets.begin(), cache.offsets.end(), p->offsets);
  if (same) {
    std::memcpy(a.a_re, cache.a_re, sizeof(a.a_re));
    std::memcpy(a.a_im, cache.a_im, sizeof(a.a_im));
    const int total = n_centers * tri::fold::kBands;
    tri::fold::fold_kernel<<<(total + tri::fold::kThreads - 1) / tri::fold::kThreads, tri::fold::kThreads, 0, s>>>(a);
    return;
  }
  for (int f = 0; f < tri::fold::kBands; ++f) {
    const double omega = std::pow(p->theta, -2.0 * f / TRI_HEAD_DIM);
    double c = 0.0, sn = 0.0;
    for (int t = 0; t < p->n_offsets; ++t) {
      c += std::cos(omega * p->offsets[t]);
      sn += std::sin(omega * p->offsets[t]);
    }
    c /= p->n_offsets;
    sn /= p->n_offsets;
    const double rc = std::cos(omega * p->delta0), rs = std::sin(omega * p->delta0);
    a.a_re[f] = c * rc - sn * rs;
    a.a_im[f] = sn * rc + c * rs;
  }
  cache.valid = true;
  cache.theta = p->theta;
  cache.delta0 = p->delta0;
  cache.offsets.assign(p->offsets, p->offsets + p->n_offsets);
  std::memcpy(cache.a_re, a.a_re, sizeof(a.a_re));
  std::memcpy(cache.a_im, a.a_im, sizeof(a.a_im));
  const int total = n_centers * tri::fold::kBands;
  tri::fold::fold_kernel<<<(total + tri::fold::kThreads - 1) / tri::fold::kThreads, tri::fold::kThreads, 0, s>>>(a);
}

// The per-offset fold: the schedule in the kernel parameters (a small block
// for short schedules, which launches faster than the largest).
template <int N>
void launch_fold_offsets(const tri_fold_params* p, const float* q_center, int n_centers, float* w_out,
                         cudaStream_t s) {
  static tri::fold::Args<N> a;   // parameter block: built in static storage (under the caller's lock)
  a.q = q_center;
  a.w = w_out;
  a.n_centers = n_centers;
  a.pairing = p->pairing;
  a.theta = p->theta;
  a.delta0 = p->delta0;
  a.n_offsets = p->n_offsets;
  for (int f = 0; f < tri::fold::kBands; ++f) a.omega[f] = std::pow(p->theta, -2.0 * f / TRI_HEAD_DIM);
  std::memcpy(a.offsets, p->offsets, sizeof(double) * p->n_offsets);
  const dim3 grid(p->n_offsets, (n_centers + tri::fold::kFoldCenters - 1) / tri::fold::kFoldCenters);
  tri::fold::fold_offsets_kernel<N><<<grid, dim3(tri::fold::kBands, tri::fold::kFoldRows), 0, s>>>(a);
}

// Shared by the two fold calls: checks, then one launch with the schedule in
// the kernel parameters.
tri_status launch_fold(const tri_fold_params* p, const float* q_center, int n_centers, float* w_out,
                       tri_stream_t stream, bool per_offset) {
  if (!p || !q_center || !w_out || n_centers < 1) return TRI_ERR_INVALID_ARG;
  if (p->head_dim != TRI_HEAD_DIM) return TRI_ERR_UNSUPPORTED;
  if (!p->offsets || p->n_offsets < 1) return TRI_ERR_INVALID_ARG;
  if (p->n_offsets > TRI_MAX_OFFSETS) return TRI_ERR_UNSUPPORTED;
  if (!(p->theta > 0.0) || !std::isfinite(p->theta) || !std::isfinite(p->delta0)) return TRI_ERR_INVALID_ARG;
  if (p->pairing != TRI_PAIRING_HALF && p->pairing != TRI_PAIRING_INTERLEAVED) return TRI_ERR_INVALID_ARG;
  for (int t = 0; t < p->n_offsets; ++t)
    if (!std::isfinite(p->offsets[t])) return TRI_ERR_INVALID_ARG;
  if (!aligned16(q_center) || !aligned16(w_out)) return TRI_ERR_INVALID_ARG;
  if (per_offset && int64_t{n_centers} * p->n_offsets > INT32_MAX / 2) return TRI_ERR_UNSUPPORTED;
  // the per-offset kernel's grid: kFoldCenters centers per block along y (at most 65535 blocks)
  if (per_offset && (int64_t{n_centers} + tri::fold::kFoldCenters - 1) / tri::fold::kFoldCenters > 65535)
    return TRI_ERR_UNSUPPORTED;
  if (int64_t{n_centers} * TRI_HEAD_DIM > INT32_MAX / 2) return TRI_ERR_UNSUPPORTED;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  tri_status st = use_device_of(q_center, &dev, &scope);
  if (st != TRI_OK) return st;
  static std::mutex m;
  std::lock_guard<std::mutex> lock(m);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!per_offset)
    launch_fold_mean(p, q_center, n_centers, w_out, s);
  else if (p->n_offsets <= tri::fold::kSmallOffsets)
    launch_fold_offsets<tri::fold::kSmallOffsets>(p, q_center, n_centers, w_out, s);
  else
    launch_fold_offsets<TRI_MAX_OFFSETS>(p, q_center, n_centers, w_out, s);
  ++g_launches;
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Rows of the key cache as one 2-D bf16 tensor [rows][128] (256-byte rows),
// when the layout packs the units back to back (CONTIG or RAGGED); 0 otherwise.
// (Sizes are checked first, so the stride products below stay in range; the
// descriptor has already passed make_geom.)
int64_t packed_rows(const tri_cache_desc* c) {
  const int64_t H = c->num_kv_heads, L = c->num_layers, Bt = c->batch;
  if (c->layout == TRI_LAYOUT_CONTIG) {
    const int64_t n = c->seq_len;
    const int64_t rows = L * H * Bt * n;               // < 2^31 * 2^30
    if (rows > INT32_MAX) return 0;
    if (Bt > 1 && c->stride_seq != n * TRI_HEAD_DIM) return 0;
    if (H > 1 && c->stride_head != Bt * n * TRI_HEAD_DIM) return 0;
    if (L > 1 && c->stride_layer != H * Bt * n * TRI_HEAD_DIM) return 0;
    return rows;
  }
  if (c->layout == TRI_LAYOUT_RAGGED) {
    const int64_t T = c->cu_seqlens[c->batch];
    const int64_t rows = L * H * T;                    // < 2^31 * 2^31
    if (T < 0 || rows > INT32_MAX) return 0;
    if (H > 1 && c->stride_head != T * TRI_HEAD_DIM) return 0;
    if (L > 1 && c->stride_layer != H * T * TRI_HEAD_DIM) return 0;
    return rows;
  }
  return 0;
}

// The key cache of a packed layout as a 2-D bf16 tensor [rows][128] for
// tiled TMA loads: boxes of 64 elements x 128 rows, 128-byte swizzle.
tri_status encode_key_map(const tri_cache_desc* desc, int64_t rows, CUtensorMap* map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return TRI_ERR_UNSUPPORTED;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(TRI_HEAD_DIM), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(tri::kRowBytes)};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(tri::score::kTileRows)};
  cuuint32_t elem[2] = {1, 1};
  CUresult cr = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(desc->k), dims, strides, box,
                       elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cr == CUDA_SUCCESS ? TRI_OK : TRI_ERR_INVALID_ARG;
}

// A PAGED key pool as a 5-D bf16 tensor for tiled TMA loads of one page:
//  * of one head (whole = false): dimensions [layer][page][token][head][128],
//    boxes of 64 elements x block_size tokens of head h;
//  * of all heads (whole = true): the token and head dimensions swapped,
//    [layer][page][head][token][128] over the same memory, boxes of 64
//    elements x block_size tokens x H heads, so that the page lands in shared
//    memory head-major (head h's tokens in consecutive rows).
// 128-byte swizzle: the same shared-memory layout as the packed map's 128-row
// boxes, a page's rows filling whole 1 KB swizzle atoms.
tri_status encode_paged_key_map(const tri_cache_desc* desc, bool whole, CUtensorMap* map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return TRI_ERR_UNSUPPORTED;
  const cuuint64_t H = static_cast<cuuint64_t>(desc->num_kv_heads);
  const cuuint64_t bs = static_cast<cuuint64_t>(desc->block_size);
  const cuuint64_t head_stride = tri::kRowBytes, token_stride = H * tri::kRowBytes;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(TRI_HEAD_DIM), whole ? bs : H, whole ? H : bs,
                        static_cast<cuuint64_t>(desc->num_blocks), static_cast<cuuint64_t>(desc->num_layers)};
  cuuint64_t strides[4] = {whole ? token_stride : head_stride, whole ? head_stride : token_stride,
                           static_cast<cuuint64_t>(desc->stride_block) * 2,
                           static_cast<cuuint64_t>(desc->stride_layer) * 2};
  cuuint32_t box[5] = {64, whole ? static_cast<cuuint32_t>(bs) : 1u,
                       whole ? static_cast<cuuint32_t>(H) : static_cast<cuuint32_t>(bs), 1, 1};
  cuuint32_t elem[5] = {1, 1, 1, 1, 1};
  CUresult cr = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(desc->k), dims, strides, box,
                       elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cr == CUDA_SUCCESS ? TRI_OK : TRI_ERR_INVALID_ARG;
}

// 128-key tiles per (layer, head), then sequence, whatever the layout (the
// max scorer's tiles); returns the tile count.
int64_t fill_head_tile_prefix(Geom* g) {
  int64_t acc = 0;
  for (int b = 0; b < g->batch; ++b) {
    g->tile_prefix[b] = static_cast<int32_t>(acc);
    acc += (g->len[b] + tri::score::kTileRows - 1) / tri::score::kTileRows;
    if (acc > INT32_MAX) return INT64_MAX;
  }
  g->tile_prefix[g->batch] = static_cast<int32_t>(acc);
  return int64_t{g->L} * g->H * acc;
}

// The max scorer's plan for a cache (host checks only, nothing launched):
// tile form, accumulator columns per head and tile count; g receives the
// tile prefix of that form.
struct MaxPlan {
  bool paged = false, whole = false;
  int head_cols = 0;      // hi and lo column of every offset, per head, rounded up to 16
  int64_t rows = 0;       // packed layouts: key rows of the [rows][128] view
  int64_t ntiles = 0;
};

tri_status plan_max(const tri_cache_desc* desc, int n_offsets, Geom* g, MaxPlan* mp) {
  if (n_offsets < 1) return TRI_ERR_INVALID_ARG;
  if (n_offsets > tri::smax::kMaxOffsets) return TRI_ERR_UNSUPPORTED;
  mp->paged = desc->layout == TRI_LAYOUT_PAGED;
  mp->head_cols = (2 * n_offsets + 15) & ~15;
  // PAGED: whole pages of all heads per tile when every head's weights fit
  // one MMA (H head_cols <= 256) and a page of all heads fills whole swizzle
  // atoms (H block_size a power of two >= 8, so whole pages fill the 128
  // rows); else one head's rows per tile, pages of a power of two >= 8 tokens.
  mp->whole = mp->paged && g->block_shift >= 0 && g->H * mp->head_cols <= tri::smax::kMaxB &&
              (g->block_size * g->H) >= 8;
  if (mp->paged) {
    if (!mp->whole && g->block_shift < 3) return TRI_ERR_UNSUPPORTED;
  } else {
    mp->rows = packed_rows(desc);
    if (mp->rows <= 0 || mp->rows > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  }
  mp->ntiles = mp->paged && !mp->whole ? fill_head_tile_prefix(g) : fill_tile_prefix(g);
  if (mp->ntiles > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  return TRI_OK;
}

// Launch the max scorer planned by plan_max (g as plan_max left it).
tri_status launch_max(const tri_cache_desc* desc, const Geom& g0, const MaxPlan& mp, const float* w, int n_offsets,
                      float* scores, int dev, cudaStream_t s) {
  if (mp.ntiles == 0) return TRI_OK;
  Geom g = g0;
  CUtensorMap map;
  tri_status st = mp.paged ? encode_paged_key_map(desc, mp.whole, &map) : encode_key_map(desc, mp.rows, &map);
  if (st != TRI_OK) return st;
#ifdef TRI_TEST_HOOKS
  g.test_skip_tile = g_test_skip_tile.load();
#endif
  const int heads = mp.whole ? g.H : 1;
  tri::smax::Args a{w, scores, static_cast<int>(mp.ntiles), n_offsets, mp.head_cols, heads, __builtin_ctz(heads),
                    mp.whole ? 1 : 0};
  const int64_t resident = int64_t{g_dev[dev].sms} * g_dev[dev].smax_blocks_per_sm;
  const int grid = static_cast<int>(mp.ntiles < resident ? mp.ntiles : resident);
  tri::smax::score_max_kernel<<<grid, tri::smax::kThreads, tri::smax::kSmemBytes, s>>>(g, map, a);
  ++g_launches;
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

}  // namespace

extern "C" {

tri_status tri_fold_weights(const tri_fold_params* p, const float* q_center, int n_centers, float* w_out,
                            tri_stream_t stream) {
  return launch_fold(p, q_center, n_centers, w_out, stream, false);
}

tri_status tri_fold_offset_weights(const tri_fold_params* p, const float* q_center, int n_centers, float* w_out,
                                   tri_stream_t stream) {
  return launch_fold(p, q_center, n_centers, w_out, stream, true);
}

tri_status tri_score_keys_max(const tri_cache_desc* desc, const float* w, int n_offsets, float* scores,
                              tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, false, &g);
  if (st != TRI_OK) return st;
  if (!w || !scores || !aligned16(w) || !aligned16(scores)) return TRI_ERR_INVALID_ARG;
  MaxPlan mp;
  st = plan_max(desc, n_offsets, &g, &mp);
  if (st != TRI_OK) return st;
  if (mp.ntiles == 0) return TRI_OK;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  return launch_max(desc, g, mp, w, n_offsets, scores, dev, reinterpret_cast<cudaStream_t>(stream));
}

tri_status tri_score_keys_at_positions(const tri_cache_desc* desc, const float* w, double theta,
                                       tri_pairing pairing, const int32_t* positions, const int64_t* query_pos,
                                       float* scores, tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, false, &g);
  if (st != TRI_OK) return st;
  if (!w || !scores || !aligned16(w) || !aligned16(scores) || !query_pos) return TRI_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !std::isfinite(theta)) return TRI_ERR_INVALID_ARG;
  if (pairing != TRI_PAIRING_HALF && pairing != TRI_PAIRING_INTERLEAVED) return TRI_ERR_INVALID_ARG;
  if (positions && !aligned16(positions)) return TRI_ERR_INVALID_ARG;
  // a page's positions are copied in 16-byte pieces from a multiple of 4 tokens
  if (positions && desc->layout == TRI_LAYOUT_PAGED && (desc->block_size % 4) != 0) return TRI_ERR_UNSUPPORTED;
  static_assert(sizeof(tri::score::Rot) + sizeof(Geom) < 32000, "kernel parameters too large");
  tri::score::Rot rot;
  std::memset(&rot, 0, sizeof(rot));
  rot.pos = positions;
  for (int b = 0; b < g.batch; ++b) {
    if (query_pos[b] < 0 || query_pos[b] > INT32_MAX) return TRI_ERR_INVALID_ARG;
    rot.qpos[b] = static_cast<int32_t>(query_pos[b]);
  }
  // C_f = omega_f / (2 pi) * 2^55, rounded (omega_f <= 1 < 2 pi, so C_f < 2^53)
  const long double two_pi = 6.283185307179586476925286766559L;
  for (int f = 0; f < tri::score::kBands; ++f) {
    const long double omega = std::pow(static_cast<long double>(theta), -2.0L * f / TRI_HEAD_DIM);
    const long double turns = omega / two_pi;
    if (!(turns >= 0.0L && turns < 1.0L)) return TRI_ERR_INVALID_ARG;
    const uint64_t c = static_cast<uint64_t>(std::llround(std::ldexp(turns, 55)));
    rot.c_hi[f] = static_cast<uint32_t>(c >> 32);
    rot.c_lo[f] = static_cast<uint32_t>(c);
  }
  const int64_t ntiles = fill_tile_prefix(&g);
  if (ntiles > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  if (ntiles == 0) return TRI_OK;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // units packed back to back: one lane per key over 2-D swizzled tiles
  const int64_t rows = desc->layout == TRI_LAYOUT_PAGED ? 0 : packed_rows(desc);
  if (rows > 0 && rows <= INT32_MAX) {
    CUtensorMap map;
    st = encode_key_map(desc, rows, &map);
    if (st != TRI_OK) return st;
    const int64_t resident = int64_t{g_dev[dev].sms} * g_dev[dev].pt_blocks_per_sm;
    const int grid = static_cast<int>(ntiles < resident ? ntiles : resident);
    if (pairing == TRI_PAIRING_HALF)
      tri::score::score_pos_tma_kernel<0><<<grid, tri::score::kPtThreads, tri::score::kPtSmemBytes, s>>>(
          g, map, rot, w, scores, static_cast<int>(ntiles));
    else
      tri::score::score_pos_tma_kernel<1><<<grid, tri::score::kPtThreads, tri::score::kPtSmemBytes, s>>>(
          g, map, rot, w, scores, static_cast<int>(ntiles));
    ++g_launches;
    TRI_CUDA(cudaGetLastError());
    return TRI_OK;
  }
  const int64_t resident = int64_t{g_dev[dev].sms} * g_dev[dev].pos_blocks_per_sm;
  const int grid = static_cast<int>(ntiles < resident ? ntiles : resident);
  if (pairing == TRI_PAIRING_HALF)
    tri::score::score_pos_kernel<0><<<grid, tri::score::kThreads, tri::score::kPosSmemBytes, s>>>(
        g, rot, w, scores, static_cast<int>(ntiles));
  else
    tri::score::score_pos_kernel<1><<<grid, tri::score::kThreads, tri::score::kPosSmemBytes, s>>>(
        g, rot, w, scores, static_cast<int>(ntiles));
  ++g_launches;
  TRI_CUDA(cudaGetLastError());
  return TRI_OK;
}

int64_t tri_score_row_stride(const tri_cache_desc* desc) {
  Geom g;
  if (make_geom(desc, false, &g) != TRI_OK) return -1;
  return g.score_stride;
}

tri_status tri_score_keys(const tri_cache_desc* desc, const float* w, float* scores, tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, false, &g);
  if (st != TRI_OK) return st;
  if (!w || !scores || !aligned16(w) || !aligned16(scores)) return TRI_ERR_INVALID_ARG;
  {
    Geom gt = g;
    if (fill_tile_prefix(&gt) > INT32_MAX) return TRI_ERR_UNSUPPORTED;
  }
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  return launch_score(g, w, scores, dev, reinterpret_cast<cudaStream_t>(stream));
}

tri_status tri_select_topk(const tri_cache_desc* desc, const float* scores, int B, int32_t* kept,
                           int32_t* kept_count, tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, false, &g);
  if (st != TRI_OK) return st;
  if (!scores || !aligned16(scores) || !kept || !kept_count || B < 1) return TRI_ERR_INVALID_ARG;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  SelectPlan plan;
  st = plan_select(g, B, &plan);
  if (st != TRI_OK) return st;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  return launch_select(g, plan, scores, B, kept, kept_count, reinterpret_cast<cudaStream_t>(stream));
}

tri_status tri_compact_kv(const tri_cache_desc* desc, const int32_t* kept, const int32_t* kept_count, int B,
                          tri_compact_mode mode, void* k_out, void* v_out, tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, true, &g);
  if (st != TRI_OK) return st;
  st = check_compact_args(desc, kept, kept_count, B, mode, k_out, v_out);
  if (st != TRI_OK) return st;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  st = check_values(desc, dev, mode, &g);
  if (st != TRI_OK) return st;
  return launch_compact(g, kept, kept_count, B, mode, k_out, v_out, dev, reinterpret_cast<cudaStream_t>(stream));
}

tri_status tri_workspace_size(const tri_cache_desc* desc, int B, size_t* bytes) {
  if (!bytes || B < 1) return TRI_ERR_INVALID_ARG;
  Geom g;
  tri_status st = make_geom(desc, false, &g);
  if (st != TRI_OK) return st;
  const int64_t units = int64_t{g.L} * g.H * g.batch;
  *bytes = static_cast<size_t>(units * g.score_stride * 4 + 256);
  return TRI_OK;
}

tri_status tri_compress(const tri_cache_desc* desc, const float* w, int B, tri_compact_mode mode, int32_t* kept,
                        int32_t* kept_count, void* k_out, void* v_out, void* workspace, size_t workspace_bytes,
                        tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, true, &g);
  if (st != TRI_OK) return st;
  if (!w || !aligned16(w)) return TRI_ERR_INVALID_ARG;
  st = check_compact_args(desc, kept, kept_count, B, mode, k_out, v_out);
  if (st != TRI_OK) return st;
  size_t need = 0;
  st = tri_workspace_size(desc, B, &need);
  if (st != TRI_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return TRI_ERR_INVALID_ARG;
  if (workspace_bytes < need) return TRI_ERR_WORKSPACE;
  SelectPlan plan;
  st = compress_checks(g, B, mode, &plan);
  if (st != TRI_OK) return st;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  st = check_values(desc, dev, mode, &g);
  if (st != TRI_OK) return st;
  return run_compress(g, plan, w, B, mode, kept, kept_count, k_out, v_out, static_cast<float*>(workspace), dev,
                      reinterpret_cast<cudaStream_t>(stream));
}

tri_status tri_compress_noalloc(const tri_cache_desc* desc, const float* w, int B, tri_compact_mode mode,
                                int32_t* kept, int32_t* kept_count, void* k_out, void* v_out, tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, true, &g);
  if (st != TRI_OK) return st;
  if (!w || !aligned16(w)) return TRI_ERR_INVALID_ARG;
  st = check_compact_args(desc, kept, kept_count, B, mode, k_out, v_out);
  if (st != TRI_OK) return st;
  const int64_t units = int64_t{g.L} * g.H * g.batch;
  if (units * g.score_stride > int64_t{TRI_NOALLOC_MAX_SCORES}) return TRI_ERR_WORKSPACE;
  SelectPlan plan;
  st = compress_checks(g, B, mode, &plan);
  if (st != TRI_OK) return st;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);   // makes the cache's device current
  if (st != TRI_OK) return st;
  st = check_values(desc, dev, mode, &g);
  if (st != TRI_OK) return st;
  float* scores = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      TRI_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scores));
      g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    scores = g_noalloc_ptr[dev];
  }
  return run_compress(g, plan, w, B, mode, kept, kept_count, k_out, v_out, scores, dev,
                      reinterpret_cast<cudaStream_t>(stream));
}

tri_status tri_compress_max(const tri_cache_desc* desc, const float* w, int n_offsets, int B,
                            tri_compact_mode mode, int32_t* kept, int32_t* kept_count, void* k_out, void* v_out,
                            void* workspace, size_t workspace_bytes, tri_stream_t stream) {
  Geom g;
  tri_status st = make_geom(desc, true, &g);
  if (st != TRI_OK) return st;
  if (!w || !aligned16(w)) return TRI_ERR_INVALID_ARG;
  st = check_compact_args(desc, kept, kept_count, B, mode, k_out, v_out);
  if (st != TRI_OK) return st;
  size_t need = 0;
  st = tri_workspace_size(desc, B, &need);
  if (st != TRI_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return TRI_ERR_INVALID_ARG;
  if (workspace_bytes < need) return TRI_ERR_WORKSPACE;
  SelectPlan plan;
  st = compress_checks(g, B, mode, &plan);
  if (st != TRI_OK) return st;
  Geom gm = g;
  MaxPlan mp;
  st = plan_max(desc, n_offsets, &gm, &mp);
  if (st != TRI_OK) return st;
  DeviceScope scope;   // the caller's current device comes back when the call returns
  int dev;
  st = use_device_of(desc->k, &dev, &scope);
  if (st != TRI_OK) return st;
  st = check_values(desc, dev, mode, &g);
  if (st != TRI_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* scores = static_cast<float*>(workspace);
  st = launch_max(desc, gm, mp, w, n_offsets, scores, dev, s);
  if (st != TRI_OK) return st;
  const bool fill = fill_in_select(g, plan, B, mode);
  st = launch_select(g, plan, scores, B, kept, kept_count, s, fill);
  if (st != TRI_OK || fill) return st;
  return launch_compact(g, kept, kept_count, B, mode, k_out, v_out, dev, s);
}

tri_status tri_read_device_status(tri_stream_t stream, uint32_t* flags, int clear) {
  if (!flags) return TRI_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceScope scope;   // the caller's current device comes back when the call returns
  if (s) {
    int dev = -1;
    TRI_CUDA(cudaStreamGetDevice(s, &dev));
    TRI_CUDA(scope.enter(dev));
  }
  unsigned int v = 0;
  TRI_CUDA(cudaMemcpyFromSymbolAsync(&v, tri::g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, s));
  TRI_CUDA(cudaStreamSynchronize(s));
  if (clear) {
    const unsigned int zero = 0;
    TRI_CUDA(cudaMemcpyToSymbolAsync(tri::g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s));
    TRI_CUDA(cudaStreamSynchronize(s));
  }
  *flags = v;
  if (v & TRI_DEVFLAG_TIMEOUT) return TRI_ERR_DEVICE_TIMEOUT;
  if (v) return TRI_ERR_DEVICE_CHECK;
  return TRI_OK;
}

const char* tri_status_string(tri_status st) {
  switch (st) {
    case TRI_OK: return "TRI_OK";
    case TRI_ERR_INVALID_ARG: return "TRI_ERR_INVALID_ARG";
    case TRI_ERR_UNSUPPORTED: return "TRI_ERR_UNSUPPORTED";
    case TRI_ERR_WORKSPACE: return "TRI_ERR_WORKSPACE";
    case TRI_ERR_CUDA: return "TRI_ERR_CUDA";
    case TRI_ERR_DEVICE_CHECK: return "TRI_ERR_DEVICE_CHECK";
    case TRI_ERR_DEVICE_TIMEOUT: return "TRI_ERR_DEVICE_TIMEOUT";
  }
  return "TRI_ERR_UNKNOWN";
}

int tri_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t tri_kernel_launches(void) { return g_launches.load(); }

const char* tri_version(void) { return "0.1.0"; }

#ifdef TRI_TEST_HOOKS
// Test builds only (not part of the product library or its header): make the
// score producer leave out one tile, so that the consumers' bounded waits run
// out and the kernel reports TRI_DEVFLAG_TIMEOUT.  -1 turns it off.
void tri_test_skip_tile(int tile) { g_test_skip_tile.store(tile); }
#endif

}  // extern "C"
