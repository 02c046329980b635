/*
 * svt.h -- C ABI of the streaming paged KV-cache attention library (libsvt.so).
 *
 * One call per step of the streaming scheme described on the pages
 *   [P1] "How Paged KV Cache Attention Enables ~20 FPS Streaming Inference in LingBot-Map"
 *   [P2] "How the Paged KV Cache Attention Mechanism Enables Long Sequence Inference in LingBot-Map"
 *   [P3] "How LingBot-Map Uses KV Caching for Efficient Streaming Inference"
 *   [P4] "How FlashInfer's Paged KV Cache Attention Outperforms SDPA Fallback in Streaming Inference"
 * Per frame step and stream: append_frame (block 0 allocates), evict_frames,
 * build_visible_page_table, plan (once per frame step), then run once per
 * transformer block ([P4] Sec. Plan-Run Execution Workflow).
 *
 * Conventions for every call:
 *  - Return value: SVT_OK (0) or a negative svt_status.  No call aborts the
 *    process; svt_last_error() returns a thread-local message for the last
 *    failure on the calling thread.  A failed call leaves the cache as it was.
 *  - Pointers named k, v, q, out, lse and opts->pool are DEVICE pointers owned
 *    by the caller; all other pointers are HOST pointers owned by the caller.
 *  - Token tensors are row-major [tokens][H][D], contiguous, in the cache dtype.
 *    A frame has Nq = num_special + page_size rows: rows 0..num_special-1 are
 *    the special tokens, the remaining page_size rows are the patch tokens.
 *  - svt_stream_t is a cudaStream_t (NULL = legacy default stream).  Device work
 *    of one cache must be issued on one CUDA stream (or ordered by the caller):
 *    kernels read the device page table written by earlier launches.  Host-side
 *    bookkeeping takes effect at call time; nothing here synchronises with the
 *    device except svt_device_error, svt_noalloc_device_error,
 *    svt_read_device_page_table and svt_selftest_wait_limit.
 *  - The library allocates its own device memory (page-table mirror, visible
 *    table, split-KV workspace, RoPE tables and scratch) once in
 *    svt_create_cache and frees it in svt_destroy_cache; svt_frame_step keeps
 *    its CUDA graphs until svt_destroy_cache.  It never frees caller memory.
 */
#ifndef SVT_H
#define SVT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVT_API __attribute__((visibility("default")))
#else
#define SVT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* svt_stream_t;
typedef struct svt_cache svt_cache;

typedef enum svt_status {
  SVT_OK = 0,
  SVT_EINVAL = -1,    /* bad argument, shape, dtype or index */
  SVT_ENOPAGES = -2,  /* a free list is empty: the pool is too small */
  SVT_ESTATE = -3,    /* call out of order (see each call) */
  SVT_ECUDA = -4,     /* a CUDA runtime/driver call failed */
  SVT_EDEVICE = -5    /* a kernel reported an out-of-range page id or a timed-out wait */
} svt_status;

typedef enum svt_dtype { SVT_BF16 = 0, SVT_FP16 = 1, SVT_FP32 = 2 } svt_dtype;

#define SVT_MAX_STREAMS 32

typedef struct svt_cache_opts {
  int num_blocks;    /* transformer blocks; each has its own pool region. Default 1. */
  int num_special;   /* special tokens per frame (camera, register, scale). Default 6.
                        [P3] Sec. Two-Stream Design: Patch and Special Tokens. Must be <= page_size. */
  int num_streams;   /* independent streams in one pool, 1..SVT_MAX_STREAMS. Default 1. */
  int dtype;         /* svt_dtype of the pool and of q, k, v and out. Default SVT_BF16. */
  int patch_pages;   /* pages reserved for the patch stream (the upstream max_num_frames);
                        pages [0, patch_pages) hold patches, [patch_pages, max_pages) specials.
                        Default num_streams*(scale_frames+sliding_window+1). */
  int max_qo_len;    /* largest total query rows of one svt_run over all streams.
                        Default num_streams*(num_special+page_size). */
  int max_splits;    /* largest number of KV chunks one (stream, head, query tile) is split
                        into by svt_plan. Default 16, range 1..64. */
  int rope_grid;     /* 0: no RoPE.  g > 0: patch tokens form a g x g grid (page_size == g*g)
                        and a 2-D RoPE is applied to patch rows of K in svt_append_frame and of
                        Q in svt_run.  [P1] Sec. Step-by-Step Streaming Inference, step 1. */
  float rope_theta;  /* RoPE base. Default 100. */
  int host_only;     /* 1: bookkeeping only -- no device memory, no kernels; k/v/q must be NULL
                        and device calls return SVT_EINVAL.  For hosts without a GPU. */
  void* pool;        /* device memory of svt_pool_bytes() bytes, 256-byte aligned, owned by
                        the caller; laid out [num_blocks][max_pages][2 (K,V)][page_tokens][H][D]
                        with page_tokens = page_size, or page_size + num_special when
                        no_cross_frame_special is set.
                        Required unless host_only.  [P4] Sec. Physical Memory Layout. */
  int no_cross_frame_special;
                     /* 0 (default): the special tokens of every frame stay visible for good
                        (kv_cache_cross_frame_special = True).  1: they leave with their frame's
                        patch tokens (kv_cache_cross_frame_special = False, [P3] Sec.
                        Configuration Parameters; Sec. Sliding-Window Eviction Strategy, "Special
                        Token Retention").  Each frame then has one page of page_size +
                        num_special tokens, its patch rows followed by its special rows ([P3]
                        Sec. The Paged KV-Cache Architecture); no special pages are used,
                        max_pages may equal patch_pages, and every visible page is full. */
} svt_cache_opts;

typedef struct svt_stats {
  int64_t frame_count;     /* frames in the stream (a provisional one included) */
  int64_t scale_pages;     /* patch pages of scale frames (never evicted) */
  int64_t live_pages;      /* patch pages in the sliding window */
  int64_t free_pages;      /* free patch pages in the pool (shared by all streams) */
  int64_t special_tokens;  /* special tokens stored for the stream */
} svt_stats;               /* [P3] Sec. Implementation Examples, "Inspecting Cache Statistics" */

typedef struct svt_plan_info {
  int num_items;                       /* attention work items of one svt_run launch */
  int splits[SVT_MAX_STREAMS];         /* KV chunks per stream (1 = no merge pass) */
  int kv_tiles[SVT_MAX_STREAMS];       /* KV tiles per stream (128 tokens at D = 64, 64 at
                                          D = 128; dense-segment tiles included) */
  int64_t kv_tokens[SVT_MAX_STREAMS];  /* visible tokens per stream (+ dense-segment rows) */
  int64_t qo_len[SVT_MAX_STREAMS];     /* query rows per stream */
} svt_plan_info;

/* Fills *opts with the defaults above (sizes that depend on the cache shape are 0 = derive). */
SVT_API void svt_default_opts(svt_cache_opts* opts);

/* Bytes of the caller-allocated pool: num_blocks*max_pages*2*page_tokens*H*D*sizeof(dtype),
 * page_tokens = page_size (+ num_special with no_cross_frame_special).
 * Returns 0 on invalid arguments.  [P2] Sec. Physical Memory Layout; [P4] Sec. Physical
 * Memory Layout (dimension 1 separates keys and values). */
SVT_API size_t svt_pool_bytes(int max_pages, int page_size, int H, int D, const svt_cache_opts* opts);

/* Creates a cache of max_pages pages of page_size tokens (page_size = patches per frame: one
 * patch page per frame, [P4] Sec. Two-Stream Design), H heads of dim D (D in {64, 128} for
 * device use), keeping scale_frames permanent frames and a window of sliding_window frames
 * ([P3] Sec. Configuration Parameters).  opts may be NULL (defaults; then host_only must be
 * given through opts, so NULL is only useful with a pool set later -- pass opts).
 * The free lists start as patch pages 0..patch_pages-1 and special pages
 * patch_pages..max_pages-1, handed out from the front.
 * Errors: SVT_EINVAL (shape, dtype, missing or misaligned pool, pool too small for
 * scale_frames+sliding_window+1 patch pages per stream), SVT_ECUDA. */
SVT_API int svt_create_cache(int max_pages, int page_size, int H, int D, int sliding_window,
                     int scale_frames, const svt_cache_opts* opts, svt_cache** out);

/* Frees the library's device and host memory (not the pool).  NULL is accepted. */
SVT_API int svt_destroy_cache(svt_cache* c);

/* Empties every stream and restores the initial free lists (the upstream clean_kv_cache,
 * [P3] Sec. The Paged KV-Cache Architecture).  Host only. */
SVT_API int svt_reset(svt_cache* c);

/* Replaces the initial free lists (a permutation of the page ids of each class).  Only on an
 * empty cache (after create or reset).  patch_ids: patch_pages ids in [0, patch_pages);
 * special_ids: max_pages-patch_pages ids in [patch_pages, max_pages).  SVT_ESTATE if not empty. */
SVT_API int svt_set_free_lists(svt_cache* c, const int32_t* patch_ids, int n_patch,
                       const int32_t* special_ids, int n_special);

/* Appends one frame's K and V ([Nq][H][D] device arrays) of transformer block `block` to
 * `stream`.  [P2] Sec. Appending New Frames; [P4] Sec. Two-Stream Design.
 * Block 0 starts a new frame: it takes one patch page from the front of the patch free list
 * (a scale page while the stream has fewer than scale_frames of them, else a window page)
 * and packs the num_special special tokens continuously after the stream's previous ones,
 * taking special pages from the special free list as pages fill.  Blocks 1..num_blocks-1
 * must then append the same frame in order; they write to the same page ids.
 * The patch rows are copied to offsets 0..page_size-1 of the patch page (with the 2-D RoPE
 * applied to K when enabled); the special rows to their (page, offset) slots.
 * If deferred eviction is on, the frame is provisional.
 * Errors: SVT_EINVAL (bad block/stream, NULL k/v on a device cache), SVT_ENOPAGES (no free
 * page; nothing changes), SVT_ESTATE (block out of order; a provisional frame not yet
 * accepted or rolled back; the window already holds more than sliding_window frames, i.e.
 * svt_evict_frames was not called after the previous append), SVT_ECUDA. */
SVT_API int svt_append_frame(svt_cache* c, int block, int stream, const void* k, const void* v,
                     svt_stream_t s);

/* Returns window pages beyond sliding_window (oldest first) to the back of the patch free
 * list.  Scale pages and special pages are never evicted.  A no-op while the last frame is
 * provisional.  Host only.  [P1] Sec. Sliding-Window Eviction Strategy; [P3] Sec.
 * Sliding-Window Eviction Strategy. */
SVT_API int svt_evict_frames(svt_cache* c, int stream);

/* Turns deferred eviction on (1) or off (0) for the stream's next appends: a frame appended
 * while it is on is provisional until svt_execute_deferred_eviction or
 * svt_rollback_last_frame.  [P3] Sec. Flow-Based Keyframe Selection. */
SVT_API int svt_set_defer_eviction(svt_cache* c, int stream, int on);

/* Accepts the provisional frame and runs the eviction it deferred.  SVT_ESTATE if there is
 * no provisional frame.  Host only. */
SVT_API int svt_execute_deferred_eviction(svt_cache* c, int stream);

/* Drops the provisional frame: its patch page goes back to the FRONT of the patch free list,
 * its special tokens are removed and any special page it opened goes back to the FRONT of
 * the special free list, so the allocator state equals the state before the append.
 * SVT_ESTATE if there is no provisional frame.  Host only. */
SVT_API int svt_rollback_last_frame(svt_cache* c, int stream);

/* Builds, on the device, the visible page table of every stream in CSR form: indptr
 * [num_streams+1], indices (per stream: scale pages in frame order, window pages oldest to
 * newest, special pages in fill order) and last_page_len [num_streams] (valid tokens on the
 * last page; only the last special page can be partial).  [P2] Sec. Building the Visible
 * Page Table; [P4] FAQ "How does the paged cache handle variable sequence lengths".
 * Reads the device page-table mirror written by the block-0 appends (same CUDA stream). */
SVT_API int svt_build_visible_page_table(svt_cache* c, svt_stream_t s);

/* Host copy of the visible page table as of the last state change (no device access).
 * capacity = length of `indices`; indptr needs num_streams+1 and last_page_len num_streams
 * entries.  *n_pages = total entries.  SVT_EINVAL if capacity is too small. */
SVT_API int svt_get_page_table(const svt_cache* c, int32_t* indptr, int32_t* indices,
                       int32_t* last_page_len, int capacity, int* n_pages);

/* Copies the DEVICE visible table (as written by the last svt_build_visible_page_table) to
 * host arrays; synchronises the stream.  For tests. */
SVT_API int svt_read_device_page_table(svt_cache* c, int32_t* indptr, int32_t* indices,
                               int32_t* last_page_len, int capacity, int* n_pages,
                               svt_stream_t s);

/* Plans the attention launch once per frame step ([P4] Sec. Plan-Run Execution Workflow):
 * qo_len_per_stream[num_streams] host array of query rows per stream (0 = stream skipped);
 * the query rows of all streams are concatenated in stream order.  A stream's query may hold
 * several frames (the first pass over a clip, [P1] Sec. Step-by-Step Streaming Inference,
 * step 1): append those frames first, then plan with their rows concatenated; with RoPE the
 * rows must be whole frames.  Splits each stream's KV
 * range into chunks so that the work items fill the GPU.  Host only; the plan is reused by
 * every block's svt_run until the cache changes.
 * Errors: SVT_ESTATE (table not rebuilt since the last change; a stream with queries but no
 * visible tokens), SVT_EINVAL (total rows > max_qo_len). */
SVT_API int svt_plan(svt_cache* c, const int32_t* qo_len_per_stream, svt_stream_t s);

/* As svt_plan, with a dense K/V segment per stream attended after its visible pages:
 * extra_len[num_streams] host array of segment rows (NULL or 0 = none; with RoPE whole frames).
 * This is the skip-append step for non-keyframes ([P1] Sec. Implementation Examples; [P3]
 * Sec. Flow-Based Keyframe Selection): the frame's queries attend to the cache plus the frame's
 * own K/V, which is never written to the pool -- the allocator, the page table and the pool
 * stay untouched.  Run the plan with svt_run_extra.  Segment rows of all streams are
 * concatenated in stream order, at most max_qo_len in total.
 * Errors: as svt_plan; SVT_EINVAL for a segment on a stream without queries. */
SVT_API int svt_plan_extra(svt_cache* c, const int32_t* qo_len_per_stream, const int32_t* extra_len,
                           svt_stream_t s);

/* Plan summary (work items, splits, tiles) for tests and benchmarks. */
SVT_API int svt_get_plan_info(const svt_cache* c, svt_plan_info* out);

/* Paged attention of block `block`: for every planned stream and query row i, head h,
 *   out[i,h,:] = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j
 * over the stream's visible tokens j (no causal mask), reading K/V through the page table.
 * [P1] Sec. FlashInfer Paged-Kernel Integration; [P2] Sec. FlashInfer Kernel Execution.
 * q, out: [sum qo_len][H][D] device arrays; out is in the cache dtype, or float32 when
 * force_fp32 != 0 or the cache dtype is SVT_FP32.  lse: NULL or [sum qo_len][H] float32
 * natural-log log-sum-exp of the scaled scores.
 * Tensor-core path (bf16/fp16 cache): scores and O accumulate in fp32 (TMEM); the softmax
 * numerators are rounded to the cache dtype before P.V and stay at or below 2^8 (fp16-safe).
 * force_fp32 = 1 computes with fp32 FMA instead of the tensor cores (the upstream's
 * force_fp32 validation path, [P2] Sec. Memory Efficiency Analysis).
 * Errors: SVT_ESTATE (no valid plan; block not yet appended for the current frame of a
 * planned stream), SVT_EINVAL, SVT_ECUDA. */
SVT_API int svt_run(svt_cache* c, int block, const void* q, void* out, float* lse, int force_fp32,
            svt_stream_t s);

/* svt_run for a plan made by svt_plan_extra: k_extra, v_extra are DEVICE [sum extra_len][H][D]
 * arrays in the cache dtype (16-byte aligned), the K and V rows of every stream's segment,
 * concatenated in stream order.  With RoPE the segment's K patch rows are rotated like
 * appended keys (into library scratch; the caller's array is not modified).  A stream with a
 * segment needs no append of the current frame in `block`.  k_extra and v_extra must be NULL
 * exactly when the plan has no segment.  Errors: as svt_run. */
SVT_API int svt_run_extra(svt_cache* c, int block, const void* q, const void* k_extra,
                          const void* v_extra, void* out, float* lse, int force_fp32, svt_stream_t s);

/* One whole frame step of one stream, from a single call: for every block b the frame's
 * k[b], v[b] are appended (svt_append_frame), then svt_evict_frames, svt_build_visible_page_table
 * and svt_plan (query rows = the frame's num_special + page_size rows on `stream`, none on the
 * others) run, then svt_run(b, q[b], out[b], lse = NULL, force_fp32 = 0) for every block.
 * k, v, q, out: HOST arrays of num_blocks DEVICE pointers.  Deferred eviction applies as set by
 * svt_set_defer_eviction.  [P1] Sec. Step-by-Step Streaming Inference; [P1] Sec. Implementation
 * Examples (the upstream captures a block's forward in a CUDA graph).
 * The appends of all blocks (num_blocks <= 64) share their page ids and run as one kernel
 * launch; the pool bytes are the same as from the separate calls.
 * use_graph = 0: the kernels are launched one by one.
 * use_graph = 1: the step's launches are recorded and issued as one CUDA graph launch.  The
 * library keeps an executable graph per launch sequence met (up to 8): the first step with a
 * new sequence builds and instantiates it, later steps give its kernel nodes the new arguments
 * (page ids, plan) and relaunch it (a graph that refuses the new arguments is rebuilt; if no
 * graph can be built the step is launched kernel by kernel).  Results are bit-identical to
 * use_graph = 0.  svt_get_graph_counts reports builds and replays.  The graphs live until
 * svt_destroy_cache; calls on one cache must come from one host thread.
 * Errors: as the calls it makes; the host bookkeeping of the sub-steps that succeeded stands
 * and their kernels are issued. */
SVT_API int svt_frame_step(svt_cache* c, int stream, const void* const* k, const void* const* v,
                           const void* const* q, void* const* out, int use_graph, svt_stream_t s);

/* Graphs built and graph replays (node updates + relaunch) by svt_frame_step so far. */
SVT_API int svt_get_graph_counts(const svt_cache* c, int* builds, int* replays);

/* Cache statistics of one stream.  [P3] Sec. Implementation Examples. */
SVT_API int svt_get_cache_stats(const svt_cache* c, int stream, svt_stats* out);

/* Synchronises `s`, reads and clears the device error word set by the kernels (page id out
 * of range, a wait that hit its limit).  Returns SVT_OK or SVT_EDEVICE (message in
 * svt_last_error). */
SVT_API int svt_device_error(svt_cache* c, svt_stream_t s);

/* Failure-detection self-test: runs a one-warp kernel that waits, with the bounded mbarrier
 * wait every kernel of this library uses, on a barrier that nothing arrives on.  The wait must
 * give up after limit_us microseconds (1..10^7) and report it; the context stays usable.
 * Synchronises `s`.  Returns SVT_EDEVICE when the wait gave up as designed (the expected
 * result), SVT_EINVAL for a bad limit, SVT_ECUDA otherwise.  The pages describe no
 * failure handling beyond rollback; this covers the kernels' own waits. */
SVT_API int svt_selftest_wait_limit(int limit_us, svt_stream_t s);

/* Paged attention for callers that cannot allocate device memory -- code running while an
 * allocator is locked or forbidden, inside a framework that owns every device buffer, or under
 * a fixed memory budget.  The paper has no counterpart: it is a variant of svt_run that needs
 * no svt_cache and takes its split-KV scratch from a fixed 32 MiB device array inside the
 * library (held by every GPU that loads the library until the process exits).  It calls no
 * cudaMalloc/cudaFree.
 * q, out: device [sum qo_len][H][D] (out in the input dtype, 16-byte aligned); lse: NULL or
 * device [sum qo_len][H] float32; pool_block: device, one block's pool region
 * [max_pages][2][page_size][H][D]; indices: DEVICE visible page ids (CSR); indptr
 * [num_streams+1], last_page_len [num_streams], qo_len [num_streams]: HOST arrays describing
 * the same table and the query rows per stream.  dtype: SVT_BF16 or SVT_FP16; D: 64 or 128.
 * num_splits: KV chunks per query tile (0 = chosen automatically within the scratch).  No 2-D
 * RoPE is applied: pass already rotated queries.
 * The first call on a device looks up the scratch array's device address (with that device
 * current); make it before any stream capture.  All calls share the scratch and calls that
 * overlap on the GPU race on it.
 * A page id outside [0, max_pages) in `indices` is read as page 0 and a wait that hits its
 * limit ends the work item early; both are recorded in a per-device error word that this
 * call does not read (it does not synchronise): call svt_noalloc_device_error.
 * Errors: SVT_EINVAL (bad argument; num_splits whose partials exceed the 32 MiB scratch),
 * SVT_ECUDA. */
SVT_API int svt_attention_noalloc(const void* q, void* out, float* lse, const void* pool_block,
                                  const int32_t* indices, const int32_t* indptr,
                                  const int32_t* last_page_len, const int32_t* qo_len,
                                  int num_streams, int max_pages, int page_size, int H, int D,
                                  int dtype, int num_splits, svt_stream_t s);

/* Synchronises `s`, then reads and clears the current device's error word of
 * svt_attention_noalloc (set by its kernels on a page id out of range or a wait that hit its
 * limit, by every call since the last read).  Allocates nothing.  The paper has no
 * counterpart.  Returns SVT_OK, SVT_EDEVICE (message in svt_last_error) or SVT_ECUDA. */
SVT_API int svt_noalloc_device_error(svt_stream_t s);

/* Message of the last failed call on this thread ("" if none). */
SVT_API const char* svt_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SVT_H */
