// svt_attention_noalloc: the paged attention of svt_run for callers that
// cannot allocate device memory -- for example code that runs while an
// allocator is locked or forbidden, inside a framework that owns every device
// buffer, or in a process whose memory budget is fixed up front.  It needs no
// svt_cache: the caller hands over the pool region, the visible page table
// and the query/output buffers.
//
// Split-KV partials (fp32 O and LSE per chunk) live in a fixed file-scope
// device array of kScratchBytes (32 MiB).  Every GPU that loads the library
// holds that array until the process exits.  The host cannot pass the
// array's name to a kernel (in host code it is only a stand-in, not a device
// address), so its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device; make that first call before any stream capture.  All calls
// share the array and it keeps the last call's contents: the attention
// kernel writes every partial before the merge reads it, so nothing needs
// clearing, but calls that overlap on the GPU (different streams, or other
// host threads) race on it.
//
// The kernels report an out-of-range page id (they read page 0 instead) or a
// wait that hit its limit in a device error word kept beside the scratch,
// one per device.  svt_noalloc_device_error reads and clears it; until then
// it keeps whatever the calls since the last read reported.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "svt_internal.h"

namespace {

using namespace svt;

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr size_t kScratchFloats = kScratchBytes / sizeof(float);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];
static __device__ __align__(256) unsigned g_noalloc_err;

std::mutex g_setup_mu;
float* g_scratch_dev[kMaxDevices] = {nullptr};
unsigned* g_err_dev[kMaxDevices] = {nullptr};

int err(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  return report_error(code, buf);
}

// Device addresses of the scratch array and error word on the current device.
int setup_device(float** scratch, unsigned** err_word) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return err(SVT_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return err(SVT_EINVAL, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_dev[dev]) {
    void* ps = nullptr;
    void* pe = nullptr;
    e = cudaGetSymbolAddress(&ps, g_noalloc_scratch);
    if (e != cudaSuccess)
      return err(SVT_ECUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    e = cudaGetSymbolAddress(&pe, g_noalloc_err);
    if (e != cudaSuccess)
      return err(SVT_ECUDA, "cudaGetSymbolAddress(error word): %s", cudaGetErrorString(e));
    g_scratch_dev[dev] = static_cast<float*>(ps);
    g_err_dev[dev] = static_cast<unsigned*>(pe);
  }
  *scratch = g_scratch_dev[dev];
  *err_word = g_err_dev[dev];
  return SVT_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

extern "C" SVT_API int svt_attention_noalloc(
    const void* q, void* out, float* lse, const void* pool_block, const int32_t* indices,
    const int32_t* indptr, const int32_t* last_page_len, const int32_t* qo_len, int num_streams,
    int max_pages, int page_size, int H, int D, int dtype, int num_splits, svt_stream_t stream) {
  if (!q || !out || !pool_block || !indices || !indptr || !last_page_len || !qo_len)
    return err(SVT_EINVAL, "null pointer argument");
  if (num_streams < 1 || num_streams > SVT_MAX_STREAMS)
    return err(SVT_EINVAL, "num_streams must be in [1, %d]", SVT_MAX_STREAMS);
  if (dtype != SVT_BF16 && dtype != SVT_FP16) return err(SVT_EINVAL, "dtype must be bf16 or fp16");
  if (!(D == 64 || D == 128) || H < 1 || page_size < 1 || max_pages < 1)
    return err(SVT_EINVAL, "unsupported shape (D must be 64 or 128)");
  if (num_splits < 0 || num_splits > 64) return err(SVT_EINVAL, "num_splits must be in [0, 64]");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out) |
       reinterpret_cast<uintptr_t>(pool_block)) % 16)
    return err(SVT_EINVAL, "q, out and pool_block must be 16-byte aligned");

  AttnParams a{};
  const int TN = attn_tile_n(D);
  const int tpp = (page_size + TN - 1) / TN;
  int rows = 0, qtiles_total = 0;
  for (int i = 0; i < num_streams; ++i) {
    const int np = indptr[i + 1] - indptr[i];
    if (qo_len[i] < 0 || np < 0 || indptr[i] < 0) return err(SVT_EINVAL, "bad qo_len or indptr");
    StreamPlan& sp = a.s[i];
    sp.q_off = rows;
    sp.nq = qo_len[i];
    sp.qtiles = (qo_len[i] + kTileM - 1) / kTileM;
    sp.page_off = indptr[i];
    sp.n_pages = np;
    sp.lpl = last_page_len[i];
    if (qo_len[i] > 0) {
      if (np == 0) return err(SVT_EINVAL, "stream %d has queries but no pages", i);
      if (sp.lpl < 1 || sp.lpl > page_size) return err(SVT_EINVAL, "last_page_len out of range");
      sp.tiles = (np - 1) * tpp + (sp.lpl + TN - 1) / TN;
    }
    rows += qo_len[i];
    qtiles_total += sp.qtiles;
  }
  if (rows == 0) return SVT_OK;
  // Split-KV chunks: enough work items for every resident CTA slot, capped
  // by the scratch size; a stream with fewer KV tiles than splits takes one
  // chunk per tile (below).
  const size_t per_split = (size_t)rows * H * (D + 1);
  const int fit = (int)std::min<size_t>(64, kScratchFloats / per_split);
  int splits = num_splits;
  if (splits > 0) {
    if (splits > 1 && (size_t)splits * per_split > kScratchFloats)
      return err(SVT_EINVAL,
                 "num_splits %d needs %zu bytes of scratch; the fixed maximum is %zu bytes "
                 "(at most %d splits for this shape)",
                 splits, (size_t)splits * per_split * sizeof(float), kScratchBytes, fit);
  } else {
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int slots = sms * attn_ctas_per_sm(D);
    const int base = H * qtiles_total;
    splits = std::max(1, (3 * slots + base - 1) / base);
    splits = std::min({splits, fit, 16});
    splits = std::max(1, splits);
  }

  float* scratch = nullptr;
  unsigned* err_word = nullptr;
  if (int r = setup_device(&scratch, &err_word)) return r;

  int items = 0;
  for (int i = 0; i < num_streams; ++i) {
    StreamPlan& sp = a.s[i];
    sp.chunks = sp.nq ? std::max(1, std::min(splits, sp.tiles)) : 0;
    sp.item_off = items;
    items += attn_items_per_stream(H, D, sp.qtiles, sp.chunks);
  }
  a.n_streams = num_streams;
  a.total_items = items;
  a.H = H;
  a.D = D;
  a.P = page_size;
  a.max_pages = max_pages;
  a.block_page_base = 0;
  a.indices = indices;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  a.out = out;
  a.lse = lse;
  a.ws_o = scratch;
  a.ws_lse = scratch + (size_t)splits * rows * H * D;
  a.ws_rows = rows;
  a.err = err_word;

  auto enc = encoder();
  if (!enc) return err(SVT_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const CUtensorMapDataType tdt =
      dtype == SVT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  alignas(64) CUtensorMap tq, tkv;
  {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kTileM};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, tdt, 3, const_cast<void*>(q), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return err(SVT_ECUDA, "cuTensorMapEncodeTiled(q) failed");
  }
  {
    cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)page_size, 2,
                          (cuuint64_t)max_pages};
    cuuint64_t strides[4] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2,
                             (cuuint64_t)page_size * H * D * 2, 2ull * page_size * H * D * 2};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)attn_tile_n(D), 1, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    if (enc(&tkv, tdt, 5, const_cast<void*>(pool_block), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return err(SVT_ECUDA, "cuTensorMapEncodeTiled(pool) failed");
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_attn_sm100(a, &tq, &tkv, nullptr, nullptr, dtype, s, nullptr);
  if (e != cudaSuccess) return err(SVT_ECUDA, "attention launch: %s", cudaGetErrorString(e));
  if (splits > 1) {
    e = launch_merge(a, dtype, s, nullptr);
    if (e != cudaSuccess) return err(SVT_ECUDA, "merge launch: %s", cudaGetErrorString(e));
  }
  return SVT_OK;
}

extern "C" SVT_API int svt_noalloc_device_error(svt_stream_t stream) {
  float* scratch = nullptr;
  unsigned* err_word = nullptr;
  if (int r = setup_device(&scratch, &err_word)) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, err_word, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(err_word, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return err(SVT_ECUDA, "read no-alloc error word: %s", cudaGetErrorString(e));
  if (h)
    return err(SVT_EDEVICE, "device error 0x%x:%s%s", h, (h & kErrPageId) ? " page-id" : "",
               (h & kErrWaitLimit) ? " wait-limit" : "");
  return SVT_OK;
}
