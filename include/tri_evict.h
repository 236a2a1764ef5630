/*
 * tri_evict.h -- C ABI of a B200 (sm_100a) library for TriAttention-style
 * KV-cache eviction: fold the offset average into one weight per band, score
 * every cached key, keep the top B keys per (layer, KV head, sequence) and
 * compact K and V to the survivors.
 *
 * Method source: the page "The future-offset average in TriAttention can be
 * precomputed" (hozhoke.com); budget default from the TriAttention README
 * (github.com/WeianMao/triattention).
 *
 * Conventions used by every call:
 *  - "device" pointers are CUDA global memory of the device that owns the
 *    cache (the library launches on the device of desc->k, or of q_center for
 *    the fold, making it current during the call only: the calling thread's
 *    current device and context are the same on return); "host" pointers are
 *    ordinary CPU memory read during the call.
 *  - The caller allocates and owns every buffer.  The library never allocates
 *    or frees device memory at run time (tri_compress_noalloc uses a fixed
 *    array of the module, allocated when the library loads) and never
 *    synchronises the stream, except tri_read_device_status, which reads a
 *    status word and waits for it.
 *  - Device calls are asynchronous on `stream` (NULL = legacy default stream).
 *    Pointers must stay valid until the stream reaches the work.
 *  - Arguments are checked on the host before anything is launched; a call
 *    that returns an error has launched nothing (TRI_ERR_CUDA excepted, which
 *    reports a launch failure).  Device code never traps: problems it can only
 *    see on the device (a page id out of range, a non-finite center, a wait
 *    that timed out) set bits in a per-device status word read by
 *    tri_read_device_status.
 *  - bf16 tensors hold IEEE binary32 values truncated to their top 16 bits
 *    (round-to-nearest-even when produced), head_dim = 128 contiguous
 *    elements per row, rows 16-byte aligned.
 *
 * A "unit" is one (layer l, KV head h, sequence b).  Units are numbered
 *     u = (l * num_kv_heads + h) * batch + b.
 * Per-unit outputs (scores, kept indices, compacted rows) are stored in that
 * order.
 */
#ifndef TRI_EVICT_H
#define TRI_EVICT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same pointer type). */
typedef struct CUstream_st* tri_stream_t;

typedef enum tri_status {
  TRI_OK = 0,
  TRI_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad alignment, inconsistent lengths */
  TRI_ERR_UNSUPPORTED = 2,    /* a valid request outside what the kernels implement (head_dim != 128, ...) */
  TRI_ERR_WORKSPACE = 3,      /* workspace smaller than tri_workspace_size() */
  TRI_ERR_CUDA = 4,           /* a CUDA runtime call failed; see tri_last_cuda_error() */
  TRI_ERR_DEVICE_CHECK = 5,   /* tri_read_device_status: a device-side check failed */
  TRI_ERR_DEVICE_TIMEOUT = 6  /* tri_read_device_status: a bounded device wait gave up */
} tri_status;

/* Which two coordinates of a head vector form rotary band f (0 <= f < d/2).
 * The page says only that the rotation turns two coordinates at a time.
 * HALF: (f, f + d/2), the rotate-half convention of Llama/Qwen checkpoints.
 * INTERLEAVED: (2f, 2f + 1). */
typedef enum tri_pairing { TRI_PAIRING_HALF = 0, TRI_PAIRING_INTERLEAVED = 1 } tri_pairing;

typedef enum tri_layout {
  /* Row (l, h, b, i) at element  l*stride_layer + h*stride_head + b*stride_seq + i*128.
   * Every sequence has seq_len keys. */
  TRI_LAYOUT_CONTIG = 0,
  /* Row (l, h, b, i) at element  l*stride_layer + h*stride_head + (cu_seqlens[b] + i)*128.
   * Sequence b has cu_seqlens[b+1] - cu_seqlens[b] keys. */
  TRI_LAYOUT_RAGGED = 1,
  /* Pages of block_size tokens, each page [block_size][num_kv_heads][128] contiguous.
   * Row (l, h, b, i) at element
   *   l*stride_layer + block_table[b*max_blocks_per_seq + i/block_size]*stride_block
   *   + (i % block_size)*num_kv_heads*128 + h*128.
   * Sequence b has seq_lens[b] keys. */
  TRI_LAYOUT_PAGED = 2
} tri_layout;

typedef enum tri_compact_mode {
  /* k_out/v_out [units][B][128]: row j of unit u is the unit's kept[u][j]-th
   * row.  Rows j >= kept_count[u] are left untouched. */
  TRI_COMPACT_OUT_OF_PLACE = 0,
  /* In place, in the cache itself ("hole fill"): in a unit with n > B keys,
   * the kept keys with index < B stay where they are, and the evicted
   * positions below B, in ascending order, receive the kept keys with index
   * >= B, in ascending order.  Afterwards the unit's first B rows are its
   * survivors; the caller shortens the sequence to B (and may release whole
   * pages past it).  Units with n <= B are not touched. */
  TRI_COMPACT_IN_PLACE_HOLEFILL = 1
} tri_compact_mode;

/* Parameters of the offline fold. */
typedef struct tri_fold_params {
  int head_dim;            /* d; must be 128 */
  double theta;            /* rotary base; omega_f = theta^(-2f/d); > 0 */
  const double* offsets;   /* HOST array: the offset schedule D (a multiset; finite values) */
  int n_offsets;           /* |D|, 1 .. TRI_MAX_OFFSETS */
  double delta0;           /* the kept distance Delta of the score, one scalar per event (0 by default) */
  tri_pairing pairing;
} tri_fold_params;

#define TRI_MAX_OFFSETS 2048
#define TRI_MAX_BATCH 256
#define TRI_HEAD_DIM 128

/* Where the cache lives.  All strides are in bf16 elements and must be
 * multiples of 8 (16 bytes).  V uses the same layout and strides as K. */
typedef struct tri_cache_desc {
  tri_layout layout;
  int num_layers;          /* L >= 1 */
  int num_kv_heads;        /* H >= 1 (PAGED: H divides 8 and block_size*H <= 128) */
  int head_dim;            /* must be 128 */
  int batch;               /* sequences, 1 .. TRI_MAX_BATCH */
  int max_seq_len;         /* capacity of a score row; 0 = the longest sequence */
  const void* k;           /* device bf16 key cache (16-byte aligned) */
  const void* v;           /* bf16 value cache on K's device; may be NULL for scoring/selection.  For an
                              OUT_OF_PLACE compaction it may instead be pinned host memory mapped into
                              the device at the same address (cudaHostAlloc): the gather then reads only
                              the kept V rows over the bus.  Anything else: TRI_ERR_INVALID_ARG. */
  int64_t stride_layer;
  int64_t stride_head;     /* CONTIG / RAGGED */
  int64_t stride_seq;      /* CONTIG */
  int64_t stride_block;    /* PAGED: elements between pages (>= block_size*H*128) */
  int seq_len;             /* CONTIG: keys per unit (>= 0) */
  const int32_t* cu_seqlens;   /* RAGGED: HOST [batch+1], cu_seqlens[0] = 0, non-decreasing */
  const int32_t* seq_lens;     /* PAGED: HOST [batch] keys per sequence */
  const int32_t* block_table;  /* PAGED: DEVICE [batch][max_blocks_per_seq] page ids */
  int max_blocks_per_seq;  /* PAGED */
  int block_size;          /* PAGED: tokens per page */
  int num_blocks;          /* PAGED: pages in the pool; ids outside [0, num_blocks) are
                              skipped on the device and flagged (TRI_ERR_DEVICE_CHECK) */
} tri_cache_desc;

/* ---------------------------------------------------------------- fold */

/* Fold the offset average into one real weight vector per center
 * (page "The future-offset average in TriAttention can be precomputed",
 * section "The averaging step - the one we improve": the offset weight
 * W_f = (1/|D|) sum_{delta in D} e^{i omega_f delta}, the offset-averaged center
 * mu'_f = E[q_f] W_f, and the real 2x2 per-band map of its closing remark).
 *
 * For each center c and band f (coordinates re(f), im(f) per `pairing`):
 *     a_f = E[q_f] * W_f * e^{i omega_f delta0},   E[q_f] = q[re] + i q[im]
 *     w[c][re(f)] = Re a_f,   w[c][im(f)] = Im a_f
 * so that for a key k, Re sum_f a_f conj(k_f) = sum_j w[j] k[j] is the
 * offset-averaged trigonometric score.  The per-band factor
 * W_f e^{i omega_f delta0} depends only on (theta, D, delta0): it is summed on
 * the host in fp64, in schedule order; the device maps every center in fp64
 * and stores fp32.
 *
 * q_center: device fp32 [n_centers][128]; w_out: device fp32 [n_centers][128].
 * Centers are indexed (l * num_kv_heads + h) by the other calls.
 * A non-finite center sets TRI_ERR_DEVICE_CHECK in the status word. */
tri_status tri_fold_weights(const tri_fold_params* params, const float* q_center,
                            int n_centers, float* w_out, tri_stream_t stream);

/* Per-offset weights for the max-over-offsets score (no averaging): for each
 * center c and offset t,
 *     a_{f,t} = E[q_f] * e^{i omega_f (delta0 + delta_t)},
 *     w_out[c][t][re(f)] = Re a_{f,t},   w_out[c][t][im(f)] = Im a_{f,t},
 * i.e. the weight vector of the literal score at distance delta0 + delta_t
 * (same page, "The same score, read as arrows in the plane").  Device fp64,
 * stored as fp32.  q_center: device fp32 [n_centers][128];
 * w_out: device fp32 [n_centers][n_offsets][128]. */
tri_status tri_fold_offset_weights(const tri_fold_params* params, const float* q_center,
                                   int n_centers, float* w_out, tri_stream_t stream);

/* ---------------------------------------------------------------- score */

/* Row stride (in floats) of the score matrix for `desc`: the longest row
 * rounded up to a multiple of 4.  Scores are [units][stride]. */
int64_t tri_score_row_stride(const tri_cache_desc* desc);

/* Score every cached key (page above, the folded form: one evaluation per key
 * instead of one per offset):
 *     scores[u][i] = sum_{j<128} w[l*H + h][j] * float(K_u[i][j])
 * an fp32 dot product of the unit's folded weight vector with the bf16 key,
 * i.e. the offset-averaged trigonometric score S~_trig of the key.
 * w: device fp32 [L*H][128] from tri_fold_weights.  scores: device fp32
 * [units][tri_score_row_stride(desc)]; entries i >= n_u are not written. */
tri_status tri_score_keys(const tri_cache_desc* desc, const float* w, float* scores,
                          tri_stream_t stream);

/* Score a pre-RoPE cache, where every key has its own distance to the query
 * (same page, "The averaging step - the one we improve", with the kept
 * distance taken per key, Delta_i = t_b - p_i, rather than one scalar):
 *     scores[u][i] = Re sum_f a_f conj(k_f) e^{i omega_f (t_b - p_i)},
 *     omega_f = theta^(-2f/128),  a_f = w[l*H + h][re(f)] + i w[l*H + h][im(f)]
 * w: device fp32 [L*H][128], the folded weights of tri_fold_weights with
 * delta0 = 0 (a nonzero delta0 adds to every key's distance).  theta and
 * pairing must be the ones the weights were folded with.
 * positions: device int32, 16-byte aligned, laid out like the scores
 * ([units][row stride], entry i of unit u is the position p_i of key i), or
 * NULL for p_i = i (a cache that has not been compacted yet); with a PAGED
 * cache, block_size must then be a multiple of 4 (else TRI_ERR_UNSUPPORTED).  query_pos: HOST int64 [batch],
 * the position t_b of the query of sequence b, 0 <= t_b < 2^31.
 * Phases are reduced exactly in fixed point and evaluated with the fp32
 * hardware sine/cosine on [-pi, pi): the result is within ~2e-6 of
 * sum_f |a_f||k_f| of the exact value.  A key with |t_b - p_i| >= 2^31 gets
 * a NaN score and sets TRI_DEVFLAG_BAD_POSITION.
 * scores: as for tri_score_keys. */
tri_status tri_score_keys_at_positions(const tri_cache_desc* desc, const float* w, double theta,
                                       tri_pairing pairing, const int32_t* positions,
                                       const int64_t* query_pos, float* scores, tri_stream_t stream);

/* Longest offset schedule tri_score_keys_max accepts. */
#define TRI_MAX_SCORE_OFFSETS 64

/* The max-over-offsets variant of the score (same page, "What it saves, and
 * what it does not": aggregating by a maximum over the offsets instead of
 * the mean; it is not linear, so it does not fold):
 *     scores[u][i] = max_{t < n_offsets} sum_j w[l*H + h][t][j] * float(K_u[i][j])
 * with w from tri_fold_offset_weights (device fp32 [L*H][n_offsets][128]).
 * More generally it is the max over any set of at most TRI_MAX_SCORE_OFFSETS
 * weight vectors per head: e.g. the offset-averaged weights of the query heads
 * of a grouped-query-attention group (n_offsets = the group size).
 * Runs on the tensor cores (bf16 keys; each fp32 weight split into two bf16
 * parts whose products accumulate in fp32, so the result keeps fp32-level
 * accuracy).  Layouts: CONTIG and RAGGED caches whose units are packed back
 * to back (stride_seq = seq_len*128, stride_head = batch*stride_seq,
 * stride_layer = H*stride_head for CONTIG; stride_head = T*128 and
 * stride_layer = H*stride_head for RAGGED with T = cu_seqlens[batch]), and
 * PAGED caches whose block_size is a power of two and where either
 * num_kv_heads * (2*n_offsets rounded up to 16) <= 256 and
 * num_kv_heads * block_size >= 8 (tiles of whole pages of all heads), or
 * block_size >= 8 (tiles of one head); a page id outside the pool sets
 * TRI_DEVFLAG_BAD_PAGE and that page's scores are not written.  Anything
 * else, or n_offsets > TRI_MAX_SCORE_OFFSETS, is TRI_ERR_UNSUPPORTED.
 * scores: as for tri_score_keys. */
tri_status tri_score_keys_max(const tri_cache_desc* desc, const float* w, int n_offsets, float* scores,
                              tri_stream_t stream);

/* ---------------------------------------------------------------- select */

/* Keep the highest-scoring keys (same page, opening section: the cache keeps
 * the highest-scoring keys within a budget; the budget B is TriAttention's KV
 * budget, default 2048).  Per unit with n keys: the top min(B, n) keys in the
 * order (score descending, index ascending), NaN ranked lowest and -0 equal to
 * +0, written as ASCENDING key indices to kept[u][0 .. min(B,n)), and
 * kept_count[u] = min(B, n).  Entries past kept_count are not written.
 * scores: device fp32 [units][tri_score_row_stride(desc)].
 * kept: device int32 [units][B]; kept_count: device int32 [units].
 * B >= 1.  Needs no workspace.  Rows of at most 4096 keys (a cache
 * re-compressed every window of generated tokens holds rows of B + the
 * window) are selected by one warp each, longer rows by one CTA each; both
 * give the same result.  A row too long for the CTA's shared memory (more
 * than about 655,000 keys at B = 2048) is TRI_ERR_UNSUPPORTED. */
tri_status tri_select_topk(const tri_cache_desc* desc, const float* scores, int B,
                           int32_t* kept, int32_t* kept_count, tri_stream_t stream);

/* ---------------------------------------------------------------- compact */

/* Compact K and V to the kept keys (bit copies): after scoring, the cache
 * keeps its highest-scoring keys and evicts the rest (page "The future-offset
 * average in TriAttention can be precomputed", opening section).  The page
 * does not say where the survivors go; the two layouts of tri_compact_mode
 * are this library's reading: ascending order out of place, and a hole fill
 * in place that moves the fewest rows (attention does not depend on the slot
 * order when a key's K and V rows move together).  kept / kept_count as written by tri_select_topk with the
 * same desc and B.  OUT_OF_PLACE: k_out, v_out device bf16 [units][B][128]
 * (16-byte aligned).  IN_PLACE_HOLEFILL: k_out and v_out must be NULL; the
 * cache (desc->k, desc->v) is modified, so they must point to writable
 * memory.  desc->v must be non-NULL. */
tri_status tri_compact_kv(const tri_cache_desc* desc, const int32_t* kept,
                          const int32_t* kept_count, int B, tri_compact_mode mode,
                          void* k_out, void* v_out, tri_stream_t stream);

/* ---------------------------------------------------------------- fused */

/* Bytes of workspace tri_compress needs for `desc` (the score matrix). */
tri_status tri_workspace_size(const tri_cache_desc* desc, int B, size_t* bytes);

/* score -> select -> compact in one call (no host sync): one pruning event of
 * the page above -- every cached key scored with the folded weights ("The
 * averaging step - the one we improve"), the highest-scoring keys within the
 * budget kept and the rest evicted (opening section) -- with the survivors
 * laid out as tri_compact_mode describes.  Same arguments and results as the
 * three calls; the scores live in `workspace` (device, >= tri_workspace_size
 * bytes, 256-byte aligned).  Every check of the three stages is made before
 * the first launch.
 * A CONTIG or RAGGED cache compacted OUT_OF_PLACE whose units fit one wave of
 * thread-block clusters (units x 16 CTAs <= the SM count) and whose rows hold
 * at most 8192 keys runs as ONE kernel: a cluster per unit scores its keys into
 * shared memory, selects across the cluster and copies the kept rows; its
 * scores, kept indices and compacted rows are identical, bit for bit, to the
 * three-kernel path's.
 * IN_PLACE_HOLEFILL on rows of at most 4096 keys that each move at most 512
 * rows (n - B <= 512: a serving cache re-compressed every window of new
 * tokens) runs as TWO kernels: the scorer, then the selection with one warp
 * per row, which fills the row's holes right after selecting it; kept,
 * kept_count and the cache end up as the three calls leave them.  Every other
 * case takes the three kernels. */
tri_status tri_compress(const tri_cache_desc* desc, const float* w, int B,
                        tri_compact_mode mode, int32_t* kept, int32_t* kept_count,
                        void* k_out, void* v_out, void* workspace, size_t workspace_bytes,
                        tri_stream_t stream);

/* The three steps of tri_compress with the max-over-offsets score of
 * tri_score_keys_max in place of the folded one (same page: "What it saves,
 * and what it does not" for the score, which does not fold; opening section
 * for keeping the highest-scoring keys and evicting the rest):
 * w and n_offsets as for tri_score_keys_max (device fp32
 * [L*H][n_offsets][128], from tri_fold_offset_weights); B, mode, kept,
 * kept_count, k_out, v_out, the workspace (tri_workspace_size bytes, 256-byte
 * aligned; it receives the score matrix), the results and the errors as for
 * tri_compress, and the layouts those tri_score_keys_max takes.  Runs the max
 * scorer, then the selection (in place, on rows that move at most 512 keys,
 * with the hole fill in the same warp) and the compaction; every check is made
 * on the host before the first launch. */
tri_status tri_compress_max(const tri_cache_desc* desc, const float* w, int n_offsets, int B,
                            tri_compact_mode mode, int32_t* kept, int32_t* kept_count, void* k_out, void* v_out,
                            void* workspace, size_t workspace_bytes, tri_stream_t stream);

/* ---------------------------------------------------------------- no allocation */

/* Capacity, in floats, of the built-in score scratch of tri_compress_noalloc
 * (16 MiB per device). */
#define TRI_NOALLOC_MAX_SCORES (4 * 1024 * 1024)

/* tri_compress without a caller-provided workspace.  The pages have no
 * counterpart of this call: it exists for callers that cannot allocate
 * device memory where they compress -- for instance a serving engine that
 * hands nearly all free HBM to its KV-cache pool at start-up (a new
 * cudaMalloc would fail or force cache blocks out), or a latency-critical
 * loop that cannot take cudaMalloc's implicit device synchronisation.
 *
 * Same arguments, computation and results as tri_compress, except that the
 * score matrix is kept in a fixed scratch array compiled into the library
 * (TRI_NOALLOC_MAX_SCORES floats, 256-byte aligned, held by every device
 * that loads the library until the process exits).  The call allocates and
 * frees nothing.
 *  - Limit: units * tri_score_row_stride(desc) must not exceed
 *    TRI_NOALLOC_MAX_SCORES; larger requests return TRI_ERR_WORKSPACE
 *    before anything is launched (split the cache, e.g. by layers).
 *  - Set-up: the first call on a device looks up the scratch array's device
 *    address (cudaGetSymbolAddress) with that device current; make that
 *    first call before any stream capture.  The array belongs to the
 *    library's module, which the CUDA runtime loads on a device the first
 *    time any tri_* call uses that device (lazy module loading, the default);
 *    a caller that will hand nearly all free memory to its own pool should
 *    make its first library call on each device (for instance this one, on a
 *    small cache) before it takes that memory, or the module load can fail.
 *  - Sharing: every call on a device uses the same scratch array, and it
 *    keeps the last call's contents (nothing in it needs to start at zero).
 *    Calls that overlap on the GPU -- on different streams, or from several
 *    host threads -- race on it: order them (one stream, or events). */
tri_status tri_compress_noalloc(const tri_cache_desc* desc, const float* w, int B, tri_compact_mode mode,
                                int32_t* kept, int32_t* kept_count, void* k_out, void* v_out,
                                tri_stream_t stream);

/* ---------------------------------------------------------------- status */

/* Device-side status bits (OR-ed by kernels). */
#define TRI_DEVFLAG_BAD_PAGE      0x1u  /* a page id outside [0, num_blocks) was skipped */
#define TRI_DEVFLAG_NONFINITE     0x2u  /* a non-finite center or offset in the fold */
#define TRI_DEVFLAG_TIMEOUT       0x4u  /* a bounded wait inside a kernel gave up */
#define TRI_DEVFLAG_BAD_KEPT      0x8u  /* compaction met a kept index outside [0, n) */
#define TRI_DEVFLAG_BAD_POSITION  0x10u /* a key's distance t - p fell outside (-2^31, 2^31); its score is NaN */
#define TRI_DEVFLAG_INVARIANT     0x20u /* only in a library built with -DTRI_CHECKED: a selection or compaction
                                           invariant failed (a unit's kept count is not min(B, n), a histogram
                                           does not total the row, holes and movers of a hole fill differ) */

/* Wait for `stream`, then read the status word of the device that owns
 * `stream` (the current device for NULL) into *flags, and zero it if `clear`.
 * Returns TRI_ERR_DEVICE_TIMEOUT if the timeout bit is set, else
 * TRI_ERR_DEVICE_CHECK if any bit is set, else TRI_OK. */
tri_status tri_read_device_status(tri_stream_t stream, uint32_t* flags, int clear);

/* Human-readable name of a status code (static string). */
const char* tri_status_string(tri_status status);

/* The cudaError_t behind the most recent TRI_ERR_CUDA on this thread (0 if none). */
int tri_last_cuda_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t tri_kernel_launches(void);

/* Library version, e.g. "0.1.0". */
const char* tri_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TRI_EVICT_H */
