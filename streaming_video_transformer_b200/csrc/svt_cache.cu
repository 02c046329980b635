// Host side of the streaming paged KV-cache library: the C ABI, the page
// allocator with its free lists, the device page-table mirror, the planner
// and the launches.
//
// The allocator follows the two-stream design of the pages:
//  * patch stream: one page per frame, handed out from the front of a FIFO
//    free list; the first scale_frames pages of a stream are permanent scale
//    pages, later ones enter a sliding window of sliding_window frames and
//    are returned to the back of the free list when they leave it.
//    ("How LingBot-Map Uses KV Caching for Efficient Streaming Inference",
//    Sec. Sliding-Window Eviction Strategy; "How FlashInfer's Paged KV Cache
//    Attention Outperforms SDPA Fallback in Streaming Inference", Sec.
//    Two-Stream Design.)
//  * special stream: num_special tokens per frame packed continuously over
//    pages of the same size, never evicted (same sections).  Without
//    cross-frame special retention (kv_cache_cross_frame_special = False,
//    "How LingBot-Map Uses KV Caching ...", Sec. Configuration Parameters)
//    a frame's special tokens follow its patch tokens in the frame's own page
//    and leave with it; there are no special pages then.
//  * deferred eviction and rollback of the provisional frame ("How LingBot-Map
//    Uses KV Caching ...", Sec. Flow-Based Keyframe Selection): rollback puts
//    the pages back at the FRONT of their free lists so that the allocator
//    state is exactly the state before the append.
//
// Device state kept by the library: a mirror of each stream's scale list,
// window ring and special-page list, written by the block-0 append kernel
// (page ids travel as kernel arguments, no host->device copies), from which
// the builder kernel assembles the visible page table.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <mutex>
#include <queue>
#include <string>
#include <vector>

#include "svt_internal.h"

using namespace svt;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SVT_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

int elem_size(int dtype) { return dtype == SVT_FP32 ? 4 : 2; }

struct StreamState {
  std::vector<int> scale;          // scale pages, frame order
  std::deque<int> window;          // window pages, oldest -> newest
  int ring_head = 0;               // device ring slot of window.front()
  std::vector<int> special_pages;  // fill order
  int64_t special_tokens = 0;
  int64_t frame_count = 0;
  bool defer = false;
  bool has_prov = false;           // last frame is provisional
  bool prov_scale = false;
  int prov_new_sp = 0;             // special pages opened by the provisional frame
  int blocks_done = 0;             // blocks that appended the current frame
  int cur_patch = -1;              // pages of the current frame (for blocks > 0)
  int cur_sp_off0 = 0;
  int cur_n_sp = 0;
  int cur_sp[kMaxSpecialSpan] = {0};
};

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

struct svt_cache {
  // shape and options
  int max_pages = 0, P = 0, H = 0, D = 0, W = 0, S = 0;
  int L = 1, ns = 6, n_streams = 1, dtype = SVT_BF16, elem = 2;
  bool frame_special = false;  // specials stored in the frame's page (no cross-frame retention)
  int page_tokens = 0;         // tokens per pool page: P, or P + ns with frame_special
  int patch_pages = 0, max_qo = 0, max_splits = 16, rope_grid = 0;
  float rope_theta = 100.f;
  bool host_only = false;
  bool debug_kv = false;
  int num_sms = 148;
  char* pool = nullptr;

  // allocator
  std::deque<int> patch_free, special_free;
  std::vector<int> init_patch, init_special;
  std::vector<StreamState> st;
  bool dirty = true;       // state changed since the last table build
  uint64_t version = 0;    // bumps on every build

  // plan
  bool plan_valid = false;
  uint64_t plan_version = 0;
  int total_rows = 0;
  int extra_rows = 0;      // rows of the dense K/V segments of the plan
  bool any_split = false;
  AttnParams attn{};
  SimtParams simt{};
  svt_plan_info info{};

  // device memory (one allocation)
  void* dmem = nullptr;
  int* d_scale = nullptr;
  int* d_ring = nullptr;
  int* d_special = nullptr;
  int* d_indptr = nullptr;
  int* d_indices = nullptr;
  int* d_lpl = nullptr;
  unsigned* d_err = nullptr;
  float* d_ws_o = nullptr;
  float* d_ws_lse = nullptr;
  char* d_qrope = nullptr;
  char* d_krope = nullptr;     // RoPE'd K of the dense segments
  float2* d_rope_tab = nullptr;
  int ring_cap = 1, sp_cap = 0, indices_cap = 0;

  alignas(64) CUtensorMap tmap_kv;
  bool has_tmap = false;
  alignas(64) CUtensorMap tmap_q;
  const void* tmap_q_ptr = nullptr;
  int tmap_q_rows = -1;
  alignas(64) CUtensorMap tmap_ke, tmap_ve;   // dense K/V segments (box of TN rows)

  // frame steps replayed as CUDA graphs (svt_frame_step): the launches of a
  // step are recorded into `rec` instead of being issued, then handed to an
  // executable graph whose kernel nodes are given the new arguments.
  Recorder* rec = nullptr;
  // svt_frame_step gathers the appends of all blocks here and launches them
  // together (nullptr: each svt_append_frame launches its own kernel).
  AppendBatch* batch = nullptr;
  struct StepGraph {
    std::vector<const void*> funcs;       // kernel of each node, in launch order
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    std::vector<cudaGraphNode_t> nodes;
  };
  std::vector<StepGraph> graphs;          // one per launch sequence met so far
  int graph_builds = 0, graph_replays = 0;
};

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int page_valid_tokens_last(const svt_cache* c, const StreamState& s) {
  if (!s.special_pages.empty()) return int((s.special_tokens - 1) % c->P) + 1;
  if (!s.scale.empty() || !s.window.empty()) return c->page_tokens;
  return 0;
}

int n_visible_pages(const StreamState& s) {
  return int(s.scale.size() + s.window.size() + s.special_pages.size());
}

void mark_dirty(svt_cache* c) {
  c->dirty = true;
  c->plan_valid = false;
}

int check_stream(const svt_cache* c, int stream) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  if (stream < 0 || stream >= c->n_streams)
    return fail(SVT_EINVAL, "stream %d out of range [0,%d)", stream, c->n_streams);
  return SVT_OK;
}

void debug_stats(const svt_cache* c, int stream, const char* when) {
  if (!c->debug_kv) return;
  const StreamState& s = c->st[stream];
  fprintf(stderr,
          "[svt] %s stream=%d frame_count=%lld scale_pages=%zu live_pages=%zu free_pages=%zu "
          "special_tokens=%lld\n",
          when, stream, (long long)s.frame_count, s.scale.size(), s.window.size(),
          c->patch_free.size(), (long long)s.special_tokens);
}

int encode_kv_map(svt_cache* c) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(SVT_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const cuuint64_t e = c->elem;
  const cuuint64_t pt = (cuuint64_t)c->page_tokens;
  cuuint64_t dims[5] = {(cuuint64_t)c->D, (cuuint64_t)c->H, pt, 2,
                        (cuuint64_t)c->L * (cuuint64_t)c->max_pages};
  cuuint64_t strides[4] = {c->D * e, (cuuint64_t)c->H * c->D * e, pt * c->H * c->D * e,
                           2ull * pt * c->H * c->D * e};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)attn_tile_n(c->D), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(&c->tmap_kv,
                   c->dtype == SVT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   5, c->pool, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVT_ECUDA, "cuTensorMapEncodeTiled(pool) failed: %d", (int)r);
  c->has_tmap = true;
  return SVT_OK;
}

// Tensor map over a dense [rows][H][D] array with boxes of box_rows rows.
int encode_rows_map(const svt_cache* c, CUtensorMap* map, const void* base, int rows,
                    int box_rows, const char* what) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(SVT_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const cuuint64_t e = c->elem;
  cuuint64_t dims[3] = {(cuuint64_t)c->D, (cuuint64_t)c->H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {c->D * e, (cuuint64_t)c->H * c->D * e};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map,
                   c->dtype == SVT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVT_ECUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return SVT_OK;
}

int encode_q_map(svt_cache* c, const void* q, int rows) {
  if (c->tmap_q_ptr == q && c->tmap_q_rows == rows) return SVT_OK;
  if (int r = encode_rows_map(c, &c->tmap_q, q, rows, kTileM, "q")) return r;
  c->tmap_q_ptr = q;
  c->tmap_q_rows = rows;
  return SVT_OK;
}

void fill_rope_table(const svt_cache* c, std::vector<float2>& tab) {
  // (cos, sin) of pos * theta^(-2i/m), m = D/2, i < m/2, pos < grid: angle,
  // cosine and sine in double precision, each value rounded once to fp32.
  const int m = c->D / 2, half = m / 2;
  tab.resize((size_t)c->rope_grid * half);
  for (int pos = 0; pos < c->rope_grid; ++pos)
    for (int i = 0; i < half; ++i) {
      double ang = pos * std::pow((double)c->rope_theta, -2.0 * i / m);
      tab[(size_t)pos * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
}

// ------------------------------------------------------------------ planner
// Estimated makespan (us) of a list-scheduled launch: items are handed to the
// SMs in blockIdx order as SMs become free.
double simulate(const std::vector<double>& item_cost, int num_sms) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> sm;
  for (int i = 0; i < num_sms; ++i) sm.push(0.0);
  double end = 0;
  for (double cst : item_cost) {
    double t = sm.top();
    sm.pop();
    t += cst;
    end = std::max(end, t);
    sm.push(t);
  }
  return end;
}

cudaKernelNodeParams node_params(const LaunchRecord& r, std::vector<void*>& argv) {
  argv = r.argv();
  cudaKernelNodeParams kp{};
  kp.func = const_cast<void*>(r.func);
  kp.gridDim = r.grid;
  kp.blockDim = r.block;
  kp.sharedMemBytes = r.smem;
  kp.kernelParams = argv.data();
  kp.extra = nullptr;
  return kp;
}

// Issues recorded launches one by one (the path a failed step takes, so that
// the device state follows the host bookkeeping done before the failure).
cudaError_t issue_directly(const Recorder& rec, cudaStream_t s) {
  for (const auto& r : rec.launches) {
    std::vector<void*> argv = r.argv();
    cudaError_t e = cudaLaunchKernel(r.func, r.grid, r.block, argv.data(), r.smem, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

namespace svt {
// Records a message for svt_last_error() from another translation unit.
int report_error(int code, const char* msg) {
  g_err = msg;
  return code;
}
}  // namespace svt

// =================================================================== C ABI
extern "C" {

const char* svt_last_error(void) { return g_err.c_str(); }

void svt_default_opts(svt_cache_opts* o) {
  if (!o) return;
  std::memset(o, 0, sizeof(*o));
  o->num_blocks = 1;
  o->num_special = 6;
  o->num_streams = 1;
  o->dtype = SVT_BF16;
  o->max_splits = 16;
  o->rope_theta = 100.f;
}

size_t svt_pool_bytes(int max_pages, int page_size, int H, int D, const svt_cache_opts* opts) {
  svt_cache_opts o;
  if (opts) o = *opts; else svt_default_opts(&o);
  if (max_pages <= 0 || page_size <= 0 || H <= 0 || D <= 0 || o.num_blocks <= 0) return 0;
  if (o.dtype < SVT_BF16 || o.dtype > SVT_FP32) return 0;
  const int ns = o.num_special < 0 ? 0 : o.num_special;
  const size_t page_tokens = (size_t)page_size + (o.no_cross_frame_special ? ns : 0);
  return (size_t)o.num_blocks * max_pages * 2 * page_tokens * H * D * elem_size(o.dtype);
}

int svt_create_cache(int max_pages, int page_size, int H, int D, int sliding_window,
                     int scale_frames, const svt_cache_opts* opts, svt_cache** out) {
  if (!out) return fail(SVT_EINVAL, "out is NULL");
  *out = nullptr;
  svt_cache_opts o;
  if (opts) o = *opts; else svt_default_opts(&o);
  if (o.num_blocks <= 0) o.num_blocks = 1;
  if (o.num_streams <= 0) o.num_streams = 1;
  if (o.max_splits <= 0) o.max_splits = 16;
  if (o.rope_theta <= 0.f) o.rope_theta = 100.f;
  if (max_pages <= 0 || page_size <= 0 || H <= 0 || D <= 0)
    return fail(SVT_EINVAL, "max_pages, page_size, H, D must be positive");
  if (sliding_window < 0 || scale_frames < 0)
    return fail(SVT_EINVAL, "sliding_window and scale_frames must be >= 0");
  if (o.num_special < 0 || o.num_special > page_size)
    return fail(SVT_EINVAL, "num_special must be in [0, page_size]");
  if (o.num_streams > SVT_MAX_STREAMS)
    return fail(SVT_EINVAL, "num_streams > %d", SVT_MAX_STREAMS);
  if (o.dtype < SVT_BF16 || o.dtype > SVT_FP32) return fail(SVT_EINVAL, "bad dtype");
  if (o.max_splits > 64) return fail(SVT_EINVAL, "max_splits > 64");
  if (D % 32 != 0 || D > 256) return fail(SVT_EINVAL, "D must be a multiple of 32, <= 256");
  const int need_patch = o.num_streams * (scale_frames + sliding_window + 1);
  const int patch_pages = o.patch_pages > 0 ? o.patch_pages : need_patch;
  if (patch_pages < need_patch)
    return fail(SVT_EINVAL, "patch_pages %d < num_streams*(scale_frames+sliding_window+1) = %d",
                patch_pages, need_patch);
  if (patch_pages > max_pages || (patch_pages == max_pages && !o.no_cross_frame_special))
    return fail(SVT_EINVAL, "max_pages %d leaves no special pages after %d patch pages",
                max_pages, patch_pages);
  if (o.rope_grid < 0 || (o.rope_grid > 0 && o.rope_grid * o.rope_grid != page_size))
    return fail(SVT_EINVAL, "rope_grid^2 must equal page_size");
  if ((int64_t)o.num_blocks * max_pages >= (1ll << 31))
    return fail(SVT_EINVAL, "num_blocks*max_pages too large");
  if (!o.host_only) {
    if (!o.pool) return fail(SVT_EINVAL, "opts->pool is NULL (allocate svt_pool_bytes)");
    if (reinterpret_cast<uintptr_t>(o.pool) % 256)
      return fail(SVT_EINVAL, "pool must be 256-byte aligned");
    if (o.dtype != SVT_FP32 && !(D == 64 || D == 128))
      return fail(SVT_EINVAL, "tensor-core path supports D in {64, 128}");
    if ((size_t)H * D * elem_size(o.dtype) % 16)
      return fail(SVT_EINVAL, "H*D*elem must be a multiple of 16 bytes");
  }

  svt_cache* c = new (std::nothrow) svt_cache();
  if (!c) return fail(SVT_EINVAL, "out of host memory");
  c->max_pages = max_pages;
  c->P = page_size;
  c->H = H;
  c->D = D;
  c->W = sliding_window;
  c->S = scale_frames;
  c->L = o.num_blocks;
  c->ns = o.num_special;
  c->frame_special = o.no_cross_frame_special != 0;
  c->page_tokens = page_size + (c->frame_special ? o.num_special : 0);
  c->n_streams = o.num_streams;
  c->dtype = o.dtype;
  c->elem = elem_size(o.dtype);
  c->patch_pages = patch_pages;
  c->max_qo = o.max_qo_len > 0 ? o.max_qo_len : o.num_streams * (o.num_special + page_size);
  c->max_splits = o.max_splits;
  c->rope_grid = o.rope_grid;
  c->rope_theta = o.rope_theta;
  c->host_only = o.host_only != 0;
  c->pool = static_cast<char*>(o.pool);
  const char* dbg = std::getenv("SVT_DEBUG_KV");
  c->debug_kv = dbg && dbg[0] == '1';
  c->ring_cap = sliding_window + 1;
  c->sp_cap = max_pages - patch_pages;
  c->indices_cap = o.num_streams * (scale_frames + sliding_window + 1) + c->sp_cap;
  for (int i = 0; i < patch_pages; ++i) c->init_patch.push_back(i);
  for (int i = patch_pages; i < max_pages; ++i) c->init_special.push_back(i);
  c->st.resize(o.num_streams);
  for (auto& s : c->st) s.blocks_done = c->L;
  c->patch_free.assign(c->init_patch.begin(), c->init_patch.end());
  c->special_free.assign(c->init_special.begin(), c->init_special.end());

  if (!c->host_only) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) { delete c; return cuda_fail(e, "cudaDeviceGetAttribute"); }
    const int ns_ = c->n_streams;
    size_t off = 0;
    auto carve = [&](size_t bytes) { size_t at = off; off = align_up(off + bytes, 256); return at; };
    size_t o_scale = carve(sizeof(int) * ns_ * std::max(1, c->S));
    size_t o_ring = carve(sizeof(int) * ns_ * c->ring_cap);
    size_t o_special = carve(sizeof(int) * ns_ * std::max(1, c->sp_cap));
    size_t o_indptr = carve(sizeof(int) * (ns_ + 1));
    size_t o_indices = carve(sizeof(int) * c->indices_cap);
    size_t o_lpl = carve(sizeof(int) * ns_);
    size_t o_err = carve(sizeof(unsigned));
    size_t o_ws_o = carve(sizeof(float) * (size_t)c->max_splits * c->max_qo * H * D);
    size_t o_ws_lse = carve(sizeof(float) * (size_t)c->max_splits * c->max_qo * H);
    size_t o_qrope = c->rope_grid ? carve((size_t)c->max_qo * H * D * c->elem) : 0;
    size_t o_krope = c->rope_grid ? carve((size_t)c->max_qo * H * D * c->elem) : 0;
    std::vector<float2> tab;
    if (c->rope_grid) fill_rope_table(c, tab);
    size_t o_tab = c->rope_grid ? carve(sizeof(float2) * tab.size()) : 0;
    e = cudaMalloc(&c->dmem, off);
    if (e != cudaSuccess) { delete c; return cuda_fail(e, "cudaMalloc(library state)"); }
    char* b = static_cast<char*>(c->dmem);
    c->d_scale = reinterpret_cast<int*>(b + o_scale);
    c->d_ring = reinterpret_cast<int*>(b + o_ring);
    c->d_special = reinterpret_cast<int*>(b + o_special);
    c->d_indptr = reinterpret_cast<int*>(b + o_indptr);
    c->d_indices = reinterpret_cast<int*>(b + o_indices);
    c->d_lpl = reinterpret_cast<int*>(b + o_lpl);
    c->d_err = reinterpret_cast<unsigned*>(b + o_err);
    c->d_ws_o = reinterpret_cast<float*>(b + o_ws_o);
    c->d_ws_lse = reinterpret_cast<float*>(b + o_ws_lse);
    if (c->rope_grid) {
      c->d_qrope = b + o_qrope;
      c->d_krope = b + o_krope;
      c->d_rope_tab = reinterpret_cast<float2*>(b + o_tab);
    }
    e = cudaMemset(c->dmem, 0, off);
    if (e == cudaSuccess && c->rope_grid)
      e = cudaMemcpy(c->d_rope_tab, tab.data(), sizeof(float2) * tab.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(c->dmem); delete c; return cuda_fail(e, "cache init"); }
    if (c->dtype != SVT_FP32) {
      int r = encode_kv_map(c);
      if (r) { cudaFree(c->dmem); delete c; return r; }
    }
  }
  *out = c;
  return SVT_OK;
}

int svt_destroy_cache(svt_cache* c) {
  if (!c) return SVT_OK;
  for (auto& g : c->graphs) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    if (g.graph) cudaGraphDestroy(g.graph);
  }
  if (c->dmem) cudaFree(c->dmem);
  delete c;
  return SVT_OK;
}

int svt_reset(svt_cache* c) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  for (auto& s : c->st) {
    s = StreamState();
    s.blocks_done = c->L;
  }
  c->patch_free.assign(c->init_patch.begin(), c->init_patch.end());
  c->special_free.assign(c->init_special.begin(), c->init_special.end());
  mark_dirty(c);
  return SVT_OK;
}

int svt_set_free_lists(svt_cache* c, const int32_t* patch_ids, int n_patch,
                       const int32_t* special_ids, int n_special) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  for (const auto& s : c->st)
    if (s.frame_count) return fail(SVT_ESTATE, "free lists can only be set on an empty cache");
  if (n_patch != c->patch_pages || n_special != c->max_pages - c->patch_pages || !patch_ids ||
      (n_special && !special_ids))
    return fail(SVT_EINVAL, "free lists must list every page of their class");
  std::vector<char> seen(c->max_pages, 0);
  for (int i = 0; i < n_patch; ++i) {
    int p = patch_ids[i];
    if (p < 0 || p >= c->patch_pages || seen[p]) return fail(SVT_EINVAL, "bad patch page id %d", p);
    seen[p] = 1;
  }
  for (int i = 0; i < n_special; ++i) {
    int p = special_ids[i];
    if (p < c->patch_pages || p >= c->max_pages || seen[p])
      return fail(SVT_EINVAL, "bad special page id %d", p);
    seen[p] = 1;
  }
  c->init_patch.assign(patch_ids, patch_ids + n_patch);
  c->init_special.assign(special_ids, special_ids + n_special);
  return svt_reset(c);
}

int svt_append_frame(svt_cache* c, int block, int stream, const void* k, const void* v,
                     svt_stream_t cs) {
  if (int r = check_stream(c, stream)) return r;
  if (block < 0 || block >= c->L) return fail(SVT_EINVAL, "block %d out of range", block);
  if (c->host_only) {
    if (k || v) return fail(SVT_EINVAL, "host-only cache takes no k/v");
  } else if (!k || !v) {
    return fail(SVT_EINVAL, "k and v must be device pointers");
  }
  StreamState& s = c->st[stream];
  const int P = c->P, ns = c->ns;
  AppendParams ap{};
  if (block == 0) {
    if (s.blocks_done != c->L)
      return fail(SVT_ESTATE, "block 0 of a new frame before blocks %d..%d of the previous one",
                  s.blocks_done, c->L - 1);
    if (s.has_prov)
      return fail(SVT_ESTATE, "previous frame is provisional: execute_deferred_eviction or "
                              "rollback_last_frame first");
    if ((int)s.window.size() > c->W)
      return fail(SVT_ESTATE, "window holds %zu > sliding_window frames: call evict_frames "
                              "after each append", s.window.size());
    // specials: tokens [n0, n0+ns) of the stream's special sequence (in the
    // frame's own page without cross-frame retention: no special pages)
    const int64_t n0 = s.special_tokens;
    const bool packed = ns && !c->frame_special;
    const int first_pg = int(n0 / P);
    const int last_pg = packed ? int((n0 + ns - 1) / P) : first_pg - 1;
    const int n_new = packed ? std::max(0, last_pg + 1 - (int)s.special_pages.size()) : 0;
    const int n_touch = packed ? last_pg - first_pg + 1 : 0;
    if (n_touch > kMaxSpecialSpan) return fail(SVT_EINVAL, "special tokens span too many pages");
    if (c->patch_free.empty()) return fail(SVT_ENOPAGES, "patch free list is empty");
    if ((int)c->special_free.size() < n_new) return fail(SVT_ENOPAGES, "special free list is empty");
    if ((int64_t)s.special_pages.size() + n_new > c->sp_cap)
      return fail(SVT_ENOPAGES, "special page capacity exhausted");
    // allocate (no failure after this point except a launch error, which is rolled back)
    const int page = c->patch_free.front();
    c->patch_free.pop_front();
    int new_sp[kMaxSpecialSpan];
    for (int i = 0; i < n_new; ++i) {
      new_sp[i] = c->special_free.front();
      c->special_free.pop_front();
      s.special_pages.push_back(new_sp[i]);
    }
    const bool is_scale = (int)s.scale.size() < c->S;
    int slot_index;
    if (is_scale) {
      slot_index = (int)s.scale.size();
      s.scale.push_back(page);
    } else {
      slot_index = (s.ring_head + (int)s.window.size()) % c->ring_cap;
      s.window.push_back(page);
    }
    s.special_tokens += ns;
    s.frame_count += 1;
    s.has_prov = s.defer;
    s.prov_scale = is_scale;
    s.prov_new_sp = n_new;
    s.blocks_done = 0;
    s.cur_patch = page;
    s.cur_sp_off0 = packed ? int(n0 % P) : 0;
    s.cur_n_sp = n_touch;
    for (int i = 0; i < n_touch; ++i) s.cur_sp[i] = s.special_pages[first_pg + i];
    mark_dirty(c);
    if (!c->host_only) {
      ap.mirror_patch = (is_scale ? c->d_scale + (size_t)stream * std::max(1, c->S)
                                  : c->d_ring + (size_t)stream * c->ring_cap) + slot_index;
      ap.mirror_special = c->d_special + (size_t)stream * std::max(1, c->sp_cap) +
                          (s.special_pages.size() - n_new);
      ap.n_new_sp = n_new;
      for (int i = 0; i < n_new; ++i) ap.new_sp[i] = new_sp[i];
    }
  } else if (s.blocks_done != block) {
    return fail(SVT_ESTATE, "block %d appended out of order (expected block %d)", block,
                s.blocks_done == c->L ? 0 : s.blocks_done);
  }
  if (!c->host_only) {
    ap.pool_block =
        c->pool + (size_t)block * c->max_pages * 2 * c->page_tokens * c->H * c->D * c->elem;
    ap.k = static_cast<const char*>(k);
    ap.v = static_cast<const char*>(v);
    ap.ns = ns;
    ap.P = P;
    ap.page_tokens = c->page_tokens;
    ap.frame_special = c->frame_special ? 1 : 0;
    ap.H = c->H;
    ap.D = c->D;
    ap.elem = c->elem;
    ap.patch_page = s.cur_patch;
    ap.sp_off0 = s.cur_sp_off0;
    ap.n_sp = s.cur_n_sp;
    for (int i = 0; i < s.cur_n_sp; ++i) ap.sp_pages[i] = s.cur_sp[i];
    ap.rope_tab = c->rope_grid ? c->d_rope_tab : nullptr;
    ap.rope_grid = c->rope_grid;
    if (c->batch) {   // launched later, with the other blocks of this frame
      if (block == 0) c->batch->p = ap;
      c->batch->k[block] = ap.k;
      c->batch->v[block] = ap.v;
      c->batch->n_blocks = block + 1;
      s.blocks_done = block + 1;
      if (block == 0) debug_stats(c, stream, "append");
      return SVT_OK;
    }
    cudaError_t e = launch_append(ap, c->dtype, reinterpret_cast<cudaStream_t>(cs), c->rec);
    if (e != cudaSuccess) {
      if (block == 0) {  // undo the allocation so that a failed call changes nothing
        s.has_prov = true;
        svt_rollback_last_frame(c, stream);
        s.has_prov = false;
      }
      return cuda_fail(e, "append kernel launch");
    }
  }
  s.blocks_done = block + 1;
  if (block == 0) debug_stats(c, stream, "append");
  return SVT_OK;
}

int svt_evict_frames(svt_cache* c, int stream) {
  if (int r = check_stream(c, stream)) return r;
  StreamState& s = c->st[stream];
  if (s.has_prov) return SVT_OK;  // eviction deferred
  bool changed = false;
  while ((int)s.window.size() > c->W) {
    c->patch_free.push_back(s.window.front());
    s.window.pop_front();
    s.ring_head = (s.ring_head + 1) % c->ring_cap;
    if (c->frame_special) s.special_tokens -= c->ns;   // the frame's specials leave too
    changed = true;
  }
  if (changed) {
    mark_dirty(c);
    debug_stats(c, stream, "evict");
  }
  return SVT_OK;
}

int svt_set_defer_eviction(svt_cache* c, int stream, int on) {
  if (int r = check_stream(c, stream)) return r;
  c->st[stream].defer = on != 0;
  return SVT_OK;
}

int svt_execute_deferred_eviction(svt_cache* c, int stream) {
  if (int r = check_stream(c, stream)) return r;
  StreamState& s = c->st[stream];
  if (!s.has_prov) return fail(SVT_ESTATE, "no provisional frame to accept");
  s.has_prov = false;
  return svt_evict_frames(c, stream);
}

int svt_rollback_last_frame(svt_cache* c, int stream) {
  if (int r = check_stream(c, stream)) return r;
  StreamState& s = c->st[stream];
  if (!s.has_prov) return fail(SVT_ESTATE, "no provisional frame to roll back");
  for (int i = 0; i < s.prov_new_sp; ++i) {
    c->special_free.push_front(s.special_pages.back());
    s.special_pages.pop_back();
  }
  int page;
  if (s.prov_scale) {
    page = s.scale.back();
    s.scale.pop_back();
  } else {
    page = s.window.back();
    s.window.pop_back();
  }
  c->patch_free.push_front(page);
  s.special_tokens -= c->ns;
  s.frame_count -= 1;
  s.has_prov = false;
  s.prov_new_sp = 0;
  s.blocks_done = c->L;
  mark_dirty(c);
  debug_stats(c, stream, "rollback");
  return SVT_OK;
}

int svt_get_cache_stats(const svt_cache* c, int stream, svt_stats* out) {
  if (int r = check_stream(c, stream)) return r;
  if (!out) return fail(SVT_EINVAL, "out is NULL");
  const StreamState& s = c->st[stream];
  out->frame_count = s.frame_count;
  out->scale_pages = (int64_t)s.scale.size();
  out->live_pages = (int64_t)s.window.size();
  out->free_pages = (int64_t)c->patch_free.size();
  out->special_tokens = s.special_tokens;
  return SVT_OK;
}

int svt_get_page_table(const svt_cache* c, int32_t* indptr, int32_t* indices,
                       int32_t* last_page_len, int capacity, int* n_pages) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  int total = 0;
  for (const auto& s : c->st) total += n_visible_pages(s);
  if (n_pages) *n_pages = total;
  if (!indptr || !last_page_len || (total && !indices)) return fail(SVT_EINVAL, "null output");
  if (capacity < total) return fail(SVT_EINVAL, "capacity %d < %d entries", capacity, total);
  int at = 0;
  for (int i = 0; i < c->n_streams; ++i) {
    const StreamState& s = c->st[i];
    indptr[i] = at;
    for (int p : s.scale) indices[at++] = p;
    for (int p : s.window) indices[at++] = p;
    for (int p : s.special_pages) indices[at++] = p;
    last_page_len[i] = page_valid_tokens_last(c, s);
  }
  indptr[c->n_streams] = at;
  return SVT_OK;
}

int svt_build_visible_page_table(svt_cache* c, svt_stream_t cs) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  if (!c->host_only) {
    BuildParams bp{};
    bp.n_streams = c->n_streams;
    bp.S = std::max(1, c->S);
    bp.ring_cap = c->ring_cap;
    bp.sp_cap = std::max(1, c->sp_cap);
    bp.max_pages = c->max_pages;
    bp.scale = c->d_scale;
    bp.ring = c->d_ring;
    bp.special = c->d_special;
    bp.indptr = c->d_indptr;
    bp.indices = c->d_indices;
    bp.lpl = c->d_lpl;
    bp.err = c->d_err;
    for (int i = 0; i < c->n_streams; ++i) {
      const StreamState& s = c->st[i];
      bp.s[i] = BuildStream{(int)s.scale.size(), s.ring_head, (int)s.window.size(),
                            (int)s.special_pages.size(), page_valid_tokens_last(c, s)};
    }
    cudaError_t e = launch_build_table(bp, reinterpret_cast<cudaStream_t>(cs), c->rec);
    if (e != cudaSuccess) return cuda_fail(e, "table builder launch");
  }
  c->dirty = false;
  c->plan_valid = false;
  c->version += 1;
  return SVT_OK;
}

int svt_read_device_page_table(svt_cache* c, int32_t* indptr, int32_t* indices,
                               int32_t* last_page_len, int capacity, int* n_pages,
                               svt_stream_t cs) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  if (c->host_only) return fail(SVT_EINVAL, "host-only cache has no device table");
  if (!indptr || !last_page_len) return fail(SVT_EINVAL, "null output");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(cs);
  cudaError_t e = cudaMemcpyAsync(indptr, c->d_indptr, sizeof(int) * (c->n_streams + 1),
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read indptr");
  int total = indptr[c->n_streams];
  if (n_pages) *n_pages = total;
  if (total < 0 || total > c->indices_cap) return fail(SVT_EDEVICE, "device indptr corrupt");
  if (capacity < total) return fail(SVT_EINVAL, "capacity %d < %d entries", capacity, total);
  if (total) {
    if (!indices) return fail(SVT_EINVAL, "null indices");
    e = cudaMemcpyAsync(indices, c->d_indices, sizeof(int) * total, cudaMemcpyDeviceToHost, s);
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(last_page_len, c->d_lpl, sizeof(int) * c->n_streams,
                        cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read device table");
  return SVT_OK;
}

int svt_plan(svt_cache* c, const int32_t* qo_len, svt_stream_t s) {
  return svt_plan_extra(c, qo_len, nullptr, s);
}

int svt_plan_extra(svt_cache* c, const int32_t* qo_len, const int32_t* extra_len, svt_stream_t) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  if (!qo_len) return fail(SVT_EINVAL, "qo_len_per_stream is NULL");
  if (c->dirty) return fail(SVT_ESTATE, "cache changed since build_visible_page_table");
  const int P = c->P;
  const int PT = c->page_tokens;
  const int TN = attn_tile_n(c->D);
  const int tpp = (PT + TN - 1) / TN;
  int rows = 0, page_off = 0;
  AttnParams& a = c->attn;
  SimtParams& m = c->simt;
  a = AttnParams{};
  m = SimtParams{};
  svt_plan_info& info = c->info;
  info = svt_plan_info{};
  std::vector<int> tiles(c->n_streams, 0), qt(c->n_streams, 0);
  int extra_rows = 0;
  for (int i = 0; i < c->n_streams; ++i) {
    const StreamState& s = c->st[i];
    const int np = n_visible_pages(s);
    const int lpl = page_valid_tokens_last(c, s);
    const int xl = extra_len ? extra_len[i] : 0;
    if (qo_len[i] < 0 || xl < 0) return fail(SVT_EINVAL, "negative qo_len or extra_len");
    if (xl > 0 && qo_len[i] == 0) return fail(SVT_EINVAL, "stream %d: extra_len without queries", i);
    if (c->rope_grid && xl % (c->ns + P))
      return fail(SVT_EINVAL, "with RoPE each stream's extra segment is whole frames of %d rows",
                  c->ns + P);
    if (qo_len[i] > 0 && np == 0 && xl == 0)
      return fail(SVT_ESTATE, "stream %d has queries but no visible tokens", i);
    if (c->rope_grid && qo_len[i] % (c->ns + P))
      return fail(SVT_EINVAL, "with RoPE each stream's query is whole frames of %d rows", c->ns + P);
    StreamPlan& sp = a.s[i];
    sp.q_off = rows;
    sp.nq = qo_len[i];
    sp.qtiles = (qo_len[i] + kTileM - 1) / kTileM;
    sp.page_off = page_off;
    sp.n_pages = np;
    sp.lpl = lpl;
    sp.tiles = (np ? (np - 1) * tpp + (lpl + TN - 1) / TN : 0) + (xl + TN - 1) / TN;
    sp.extra_len = xl;
    sp.extra_off = extra_rows;
    extra_rows += xl;
    tiles[i] = sp.tiles;
    qt[i] = sp.qtiles;
    rows += qo_len[i];
    page_off += np;
    info.kv_tiles[i] = sp.tiles;
    info.kv_tokens[i] = (np ? (int64_t)(np - 1) * PT + lpl : 0) + xl;
    info.qo_len[i] = qo_len[i];
  }
  if (rows > c->max_qo) return fail(SVT_EINVAL, "total query rows %d > max_qo_len %d", rows, c->max_qo);
  if (extra_rows > c->max_qo)
    return fail(SVT_EINVAL, "total extra rows %d > max_qo_len %d", extra_rows, c->max_qo);
  // Choose KV splits: candidate k scales every stream's chunk count with its tile count.
  int max_tiles = 0;
  for (int i = 0; i < c->n_streams; ++i)
    if (qo_len[i]) max_tiles = std::max(max_tiles, tiles[i]);
  // Cost model: a work item is one 128-row query tile over a KV chunk; a KV
  // tile costs 4*128*TN*D flops at 6.6 TFLOP/s per SM (a round figure near
  // what the kernel sustains; only its ratio to the fixed per-item and merge
  // costs steers the choice), shared by the CTAs resident on one SM.
  const double tile_us = 4.0 * kTileM * TN * c->D / 6.6e6 * attn_ctas_per_sm(c->D);
  const double item_us = 2.0;
  const int slots = c->num_sms * attn_ctas_per_sm(c->D);
  // The KV tiles' work does not depend on the split: every chunk set covers
  // each stream's tiles once per head and query tile.
  double tile_work = 0;
  for (int i = 0; i < c->n_streams; ++i)
    if (qo_len[i]) tile_work += (double)c->H * qt[i] * tiles[i] * tile_us;
  std::vector<int> best(c->n_streams, 1);
  double best_t = 1e300;
  std::vector<double> cost;
  for (int k = 1; k <= c->max_splits; ++k) {
    std::vector<int> ch(c->n_streams, 1);
    bool split = false;
    double merge_bytes = 0, n_items = 0;
    for (int i = 0; i < c->n_streams; ++i) {
      if (!qo_len[i]) continue;
      int cc = (int)std::ceil((double)k * tiles[i] / std::max(1, max_tiles));
      cc = std::max(1, std::min({cc, c->max_splits, tiles[i]}));
      ch[i] = cc;
      n_items += (double)c->H * cc * qt[i];
      if (cc > 1) {
        split = true;
        merge_bytes += (double)qo_len[i] * c->H * (c->D + 1) * 4.0 * (cc + 1);
      }
    }
    const double merge_us = split ? 4.0 + merge_bytes / 5.0e6 : 0.0;
    // No schedule finishes before its work spread evenly over the CTA slots,
    // and that bound never falls as k grows (more items, more merge traffic):
    // once it reaches what the best split so far would have to beat, no
    // larger k can be chosen.
    if (((tile_work + n_items * item_us) / slots + merge_us) * (1.0 - 1e-9) >= best_t * 0.98) break;
    cost.clear();
    for (int i = 0; i < c->n_streams; ++i) {
      if (!qo_len[i]) continue;
      const int cc = ch[i];
      const int per_item = 1;   // one 128-row query tile per work item
      const int groups = (qt[i] + per_item - 1) / per_item;
      for (int h = 0; h < c->H; ++h)
        for (int cix = 0; cix < cc; ++cix)
          for (int g = 0; g < groups; ++g) {
            int t0 = (int)((int64_t)cix * tiles[i] / cc), t1 = (int)((int64_t)(cix + 1) * tiles[i] / cc);
            const int q_in_item = std::min(per_item, qt[i] - g * per_item);
            cost.push_back(item_us + (t1 - t0) * tile_us * q_in_item);
          }
    }
    const double t = simulate(cost, slots) + merge_us;
    if (t < best_t * 0.98) {
      best_t = t;
      best = ch;
    }
  }
  int items = 0;
  bool any_split = false;
  for (int i = 0; i < c->n_streams; ++i) {
    StreamPlan& sp = a.s[i];
    sp.chunks = qo_len[i] ? best[i] : 0;
    sp.item_off = items;
    items += attn_items_per_stream(c->H, c->D, sp.qtiles, sp.chunks);
    any_split |= sp.chunks > 1;
    info.splits[i] = sp.chunks;
  }
  a.n_streams = c->n_streams;
  a.total_items = items;
  a.H = c->H;
  a.D = c->D;
  a.P = PT;
  a.max_pages = c->max_pages;
  a.indices = c->d_indices;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c->D));
  a.ws_o = c->d_ws_o;
  a.ws_lse = c->d_ws_lse;
  a.ws_rows = c->max_qo;
  a.err = c->d_err;
  info.num_items = items;
  // fp32-FMA decomposition
  const int rb = simt_rows_per_block(c->D);
  int blocks = 0;
  m.n_streams = c->n_streams;
  for (int i = 0; i < c->n_streams; ++i) {
    SimtStream& ss = m.s[i];
    ss.q_off = a.s[i].q_off;
    ss.nq = a.s[i].nq;
    ss.rblocks = (a.s[i].nq + rb - 1) / rb;
    ss.page_off = a.s[i].page_off;
    ss.n_pages = a.s[i].n_pages;
    ss.lpl = a.s[i].lpl;
    ss.extra_len = a.s[i].extra_len;
    ss.extra_off = a.s[i].extra_off;
    ss.block_off = blocks;
    blocks += ss.rblocks * c->H;
  }
  m.total_blocks = blocks;
  m.H = c->H;
  m.D = c->D;
  m.P = PT;
  m.max_pages = c->max_pages;
  m.indices = c->d_indices;
  m.scale = (float)(1.0 / std::sqrt((double)c->D));
  m.err = c->d_err;
  c->total_rows = rows;
  c->extra_rows = extra_rows;
  c->any_split = any_split;
  c->plan_valid = true;
  c->plan_version = c->version;
  return SVT_OK;
}

int svt_get_plan_info(const svt_cache* c, svt_plan_info* out) {
  if (!c || !out) return fail(SVT_EINVAL, "null argument");
  if (!c->plan_valid) return fail(SVT_ESTATE, "no valid plan");
  *out = c->info;
  return SVT_OK;
}

int svt_run(svt_cache* c, int block, const void* q, void* out, float* lse, int force_fp32,
            svt_stream_t cs) {
  return svt_run_extra(c, block, q, nullptr, nullptr, out, lse, force_fp32, cs);
}

int svt_run_extra(svt_cache* c, int block, const void* q, const void* k_extra,
                  const void* v_extra, void* out, float* lse, int force_fp32, svt_stream_t cs) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  if (c->host_only) return fail(SVT_EINVAL, "host-only cache cannot run kernels");
  if (block < 0 || block >= c->L) return fail(SVT_EINVAL, "block %d out of range", block);
  if (!c->plan_valid || c->plan_version != c->version || c->dirty)
    return fail(SVT_ESTATE, "no valid plan for the current page table (build, then plan)");
  if (c->total_rows == 0) return SVT_OK;
  if (!q || !out) return fail(SVT_EINVAL, "q and out must be device pointers");
  if (c->extra_rows > 0 && (!k_extra || !v_extra))
    return fail(SVT_EINVAL, "the plan has dense K/V segments: pass k_extra and v_extra");
  if (c->extra_rows == 0 && (k_extra || v_extra))
    return fail(SVT_EINVAL, "the plan has no dense K/V segment (plan with extra_len)");
  for (int i = 0; i < c->n_streams; ++i)
    if (c->attn.s[i].nq && c->attn.s[i].extra_len == 0 && c->st[i].blocks_done <= block)
      return fail(SVT_ESTATE, "stream %d: block %d has not appended the current frame", i, block);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(cs);
  const char* qsrc = static_cast<const char*>(q);
  const char* ksrc = static_cast<const char*>(k_extra);
  cudaError_t e;
  if (c->rope_grid) {
    RopeQParams rp{};
    rp.q_in = qsrc;
    rp.q_out = c->d_qrope;
    rp.rows = c->total_rows;
    rp.frame_rows = c->ns + c->P;
    rp.ns = c->ns;
    rp.H = c->H;
    rp.D = c->D;
    rp.elem = c->elem;
    rp.rope_tab = c->d_rope_tab;
    rp.rope_grid = c->rope_grid;
    e = launch_rope_q(rp, c->dtype, s, c->rec);
    if (e != cudaSuccess) return cuda_fail(e, "rope_q launch");
    qsrc = c->d_qrope;
    if (c->extra_rows > 0) {   // the segment's K gets the same rotation as stored keys
      rp.q_in = ksrc;
      rp.q_out = c->d_krope;
      rp.rows = c->extra_rows;
      e = launch_rope_q(rp, c->dtype, s, c->rec);
      if (e != cudaSuccess) return cuda_fail(e, "rope_k launch");
      ksrc = c->d_krope;
    }
  }
  const size_t block_bytes = (size_t)c->max_pages * 2 * c->page_tokens * c->H * c->D * c->elem;
  if (force_fp32 || c->dtype == SVT_FP32) {
    SimtParams m = c->simt;
    m.pool_block = c->pool + (size_t)block * block_bytes;
    m.q = qsrc;
    m.k_extra = ksrc;
    m.v_extra = static_cast<const char*>(v_extra);
    m.out = static_cast<float*>(out);
    m.lse = lse;
    e = launch_attn_simt(m, c->dtype, s, c->rec);
    if (e != cudaSuccess) return cuda_fail(e, "fp32 attention launch");
    return SVT_OK;
  }
  if (reinterpret_cast<uintptr_t>(qsrc) % 16) return fail(SVT_EINVAL, "q must be 16-byte aligned");
  if (int r = encode_q_map(c, qsrc, c->total_rows)) return r;
  if (c->extra_rows > 0) {
    if ((reinterpret_cast<uintptr_t>(ksrc) | reinterpret_cast<uintptr_t>(v_extra)) % 16)
      return fail(SVT_EINVAL, "k_extra and v_extra must be 16-byte aligned");
    const int tn = attn_tile_n(c->D);
    if (int r = encode_rows_map(c, &c->tmap_ke, ksrc, c->extra_rows, tn, "k_extra")) return r;
    if (int r = encode_rows_map(c, &c->tmap_ve, v_extra, c->extra_rows, tn, "v_extra")) return r;
  }
  AttnParams a = c->attn;
  a.block_page_base = (int64_t)block * c->max_pages;
  a.out = out;
  a.lse = lse;
  e = launch_attn_sm100(a, &c->tmap_q, &c->tmap_kv, c->extra_rows ? &c->tmap_ke : nullptr,
                        c->extra_rows ? &c->tmap_ve : nullptr, c->dtype, s, c->rec);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  if (c->any_split) {
    e = launch_merge(a, c->dtype, s, c->rec);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return SVT_OK;
}

int svt_device_error(svt_cache* c, svt_stream_t cs) {
  if (!c) return fail(SVT_EINVAL, "null cache");
  if (c->host_only) return SVT_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(cs);
  unsigned h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, c->d_err, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->d_err, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (h)
    return fail(SVT_EDEVICE, "device error 0x%x:%s%s%s", h, (h & kErrPageId) ? " page-id" : "",
                (h & kErrWaitLimit) ? " wait-limit" : "", (h & kErrShape) ? " shape" : "");
  return SVT_OK;
}

int svt_frame_step(svt_cache* c, int stream, const void* const* k, const void* const* v,
                   const void* const* q, void* const* out, int use_graph, svt_stream_t cs) {
  if (int r = check_stream(c, stream)) return r;
  if (c->host_only) return fail(SVT_EINVAL, "host-only cache cannot run kernels");
  if (!k || !v || !q || !out) return fail(SVT_EINVAL, "k, v, q and out must list one pointer per block");
  for (int b = 0; b < c->L; ++b)
    if (!k[b] || !v[b] || !q[b] || !out[b]) return fail(SVT_EINVAL, "null pointer for block %d", b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(cs);
  Recorder rec;
  c->rec = use_graph ? &rec : nullptr;
  int r = SVT_OK;
  // The appends of all blocks share their page ids: one launch covers them.
  if (c->L <= kMaxBatchBlocks) {
    AppendBatch batch{};
    batch.block_bytes = (size_t)c->max_pages * 2 * c->page_tokens * c->H * c->D * c->elem;
    c->batch = &batch;
    for (int b = 0; b < c->L && !r; ++b) r = svt_append_frame(c, b, stream, k[b], v[b], cs);
    c->batch = nullptr;
    if (r && batch.n_blocks > 0) {   // a later block was refused: undo the frame's allocation
      const std::string msg = g_err;
      StreamState& st = c->st[stream];
      st.has_prov = true;
      svt_rollback_last_frame(c, stream);
      st.has_prov = false;
      g_err = msg;
    }
    if (!r) {
      cudaError_t e = launch_append_batch(batch, c->dtype, s, c->rec);
      if (e != cudaSuccess) {
        StreamState& st = c->st[stream];
        st.has_prov = true;
        svt_rollback_last_frame(c, stream);
        st.has_prov = false;
        r = cuda_fail(e, "append kernel launch");
      }
    }
  } else {
    for (int b = 0; b < c->L && !r; ++b) r = svt_append_frame(c, b, stream, k[b], v[b], cs);
  }
  if (!r) r = svt_evict_frames(c, stream);
  if (!r) r = svt_build_visible_page_table(c, cs);
  if (!r) {
    std::vector<int32_t> qo(c->n_streams, 0);
    qo[stream] = c->ns + c->P;
    r = svt_plan(c, qo.data(), cs);
  }
  for (int b = 0; b < c->L && !r; ++b) r = svt_run(c, b, q[b], out[b], nullptr, 0, cs);
  c->rec = nullptr;
  if (!use_graph || rec.launches.empty()) return r;
  if (r) {
    const std::string msg = g_err;
    issue_directly(rec, s);
    g_err = msg;
    return r;
  }
  std::vector<const void*> funcs;
  for (const auto& x : rec.launches) funcs.push_back(x.func);
  svt_cache::StepGraph* g = nullptr;
  for (auto& x : c->graphs)
    if (x.funcs == funcs) g = &x;
  std::vector<void*> argv;
  if (g) {
    bool updated = true;
    for (size_t i = 0; updated && i < rec.launches.size(); ++i) {
      cudaKernelNodeParams kp = node_params(rec.launches[i], argv);
      updated = cudaGraphExecKernelNodeSetParams(g->exec, g->nodes[i], &kp) == cudaSuccess;
    }
    if (updated) {
      c->graph_replays += 1;
    } else {                         // the executable graph refused the new arguments: rebuild it
      cudaGetLastError();
      cudaGraphExecDestroy(g->exec);
      cudaGraphDestroy(g->graph);
      c->graphs.erase(c->graphs.begin() + (g - c->graphs.data()));
      g = nullptr;
    }
  }
  if (!g) {
    if (c->graphs.size() >= 8) {     // keep a few launch sequences
      cudaGraphExecDestroy(c->graphs.front().exec);
      cudaGraphDestroy(c->graphs.front().graph);
      c->graphs.erase(c->graphs.begin());
    }
    svt_cache::StepGraph ng;
    ng.funcs = funcs;
    cudaError_t e = cudaGraphCreate(&ng.graph, 0);
    cudaGraphNode_t prev = nullptr;
    for (size_t i = 0; e == cudaSuccess && i < rec.launches.size(); ++i) {
      cudaKernelNodeParams kp = node_params(rec.launches[i], argv);
      cudaGraphNode_t node = nullptr;
      e = cudaGraphAddKernelNode(&node, ng.graph, prev ? &prev : nullptr, prev ? 1 : 0, &kp);
      ng.nodes.push_back(node);
      prev = node;
    }
    if (e == cudaSuccess) e = cudaGraphInstantiate(&ng.exec, ng.graph, 0);
    if (e != cudaSuccess) {          // no graph: the step still runs, launch by launch
      if (ng.graph) cudaGraphDestroy(ng.graph);
      cudaGetLastError();
      e = issue_directly(rec, s);
      return e == cudaSuccess ? SVT_OK : cuda_fail(e, "frame step launches");
    }
    c->graphs.push_back(std::move(ng));
    g = &c->graphs.back();
    c->graph_builds += 1;
  }
  cudaError_t e = cudaGraphLaunch(g->exec, s);
  if (e != cudaSuccess) return cuda_fail(e, "graph launch");
  return SVT_OK;
}

int svt_get_graph_counts(const svt_cache* c, int* builds, int* replays) {
  if (!c || !builds || !replays) return fail(SVT_EINVAL, "null argument");
  *builds = c->graph_builds;
  *replays = c->graph_replays;
  return SVT_OK;
}

}  // extern "C"
