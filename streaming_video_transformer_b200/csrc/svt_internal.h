// Internal declarations shared by the host library (svt_cache.cu) and the
// kernel files.  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <tuple>
#include <utility>
#include <vector>
#include <cuda_runtime.h>

#include "../../include/svt.h"

namespace svt {

// ------------------------------------------------------- kernel dispatch
// Every kernel of the library is launched through dispatch(): with no
// recorder it is launched at once (cudaLaunchKernel on the given stream);
// with a recorder the launch (function, shape, copies of the arguments) is
// appended to it instead, so that a frame step can be replayed as a CUDA
// graph whose kernel nodes take the recorded arguments.
struct LaunchRecord {
  const void* func = nullptr;
  dim3 grid, block;
  unsigned smem = 0;
  std::vector<std::shared_ptr<void>> args;   // one 64-byte aligned copy per argument
  std::vector<void*> argv() const {
    std::vector<void*> v;
    for (const auto& a : args) v.push_back(a.get());
    return v;
  }
};

struct Recorder {
  std::vector<LaunchRecord> launches;
};

namespace detail {
template <typename T>
std::shared_ptr<void> copy_arg(const T& x) {
  const size_t n = (sizeof(T) + 63) / 64 * 64;
  void* mem = std::aligned_alloc(64, n);
  if (!mem) return nullptr;
  std::memcpy(mem, &x, sizeof(T));
  return std::shared_ptr<void>(mem, [](void* q) { std::free(q); });
}
template <typename Tup, size_t... I>
void fill_argv(Tup& t, void** argv, std::index_sequence<I...>) {
  ((argv[I] = static_cast<void*>(&std::get<I>(t))), ...);
}
}  // namespace detail

template <typename... A, typename... B>
cudaError_t dispatch(Recorder* rec, void (*kern)(A...), dim3 grid, dim3 block, unsigned smem,
                     cudaStream_t s, B&&... in) {
  static_assert(sizeof...(A) == sizeof...(B), "argument count");
  std::tuple<std::decay_t<A>...> args(std::forward<B>(in)...);
  if (!rec) {
    void* argv[sizeof...(A)];
    detail::fill_argv(args, argv, std::index_sequence_for<A...>{});
    cudaError_t e = cudaLaunchKernel(reinterpret_cast<const void*>(kern), grid, block, argv, smem, s);
    return e;
  }
  LaunchRecord r;
  r.func = reinterpret_cast<const void*>(kern);
  r.grid = grid;
  r.block = block;
  r.smem = smem;
  bool ok = true;
  std::apply([&](const auto&... a) {
    ((r.args.push_back(detail::copy_arg(a)), ok = ok && r.args.back() != nullptr), ...);
  }, args);
  if (!ok) return cudaErrorMemoryAllocation;
  rec->launches.push_back(std::move(r));
  return cudaSuccess;
}

constexpr int kMaxSpecialSpan = 8;   // special pages one frame's specials can touch
constexpr int kTileM = 128;          // query rows per tensor-core tile
constexpr int kTileN = 128;          // KV tokens per tensor-core tile at D = 64
// KV tokens per tile of the tensor-core attention kernel: 128 at D = 64, 64 at
// D = 128, so that a CTA needs 256 TMEM columns and two CTAs share an SM.
__host__ __device__ constexpr int attn_tile_n(int D) { return D == 64 ? kTileN : 64; }

// Device error word bits (OR-ed by kernels, read by svt_device_error).
enum : unsigned {
  kErrPageId = 1u,      // a page id read from the device table is out of range
  kErrWaitLimit = 2u,   // an mbarrier wait hit its iteration limit
  kErrShape = 4u,       // a kernel found a shape it does not support
};

// ---------------------------------------------------------------- append
struct AppendParams {
  char* pool_block;          // pool region of this transformer block
  const char* k;             // [Nq][H][D]
  const char* v;
  int ns, P, H, D, elem;     // elem = bytes per element; P = patch rows of a frame
  int page_tokens;           // tokens per pool page (P, or P + ns with frame_special)
  int frame_special;         // 1: special rows go to the patch page after the patches
  int patch_page;
  int sp_off0;               // offset of the frame's first special token in sp_pages[0]
  int n_sp;                  // special pages touched by this frame
  int sp_pages[kMaxSpecialSpan];
  // Block-0 update of the device page-table mirror (mirror_patch == nullptr otherwise).
  int* mirror_patch;         // slot receiving patch_page
  int* mirror_special;       // first slot receiving new special pages
  int n_new_sp;
  int new_sp[kMaxSpecialSpan];
  const float2* rope_tab;    // [grid][D/4] (cos, sin), nullptr = no RoPE
  int rope_grid;
};
cudaError_t launch_append(const AppendParams& p, int dtype, cudaStream_t s, Recorder* rec);

// The appends of one frame for blocks 0..n_blocks-1 in one launch: the same
// page ids for every block (p, with the block-0 mirror update), block b's pool
// region at p.pool_block + b * block_bytes, its rows in k[b] and v[b].
constexpr int kMaxBatchBlocks = 64;
struct AppendBatch {
  AppendParams p;
  int n_blocks;
  size_t block_bytes;
  const char* k[kMaxBatchBlocks];
  const char* v[kMaxBatchBlocks];
};
cudaError_t launch_append_batch(const AppendBatch& b, int dtype, cudaStream_t s, Recorder* rec);

// ------------------------------------------------------------- RoPE on Q
struct RopeQParams {
  const char* q_in;          // [rows][H][D]
  char* q_out;
  int rows, frame_rows, ns, H, D, elem;
  const float2* rope_tab;
  int rope_grid;
};
cudaError_t launch_rope_q(const RopeQParams& p, int dtype, cudaStream_t s, Recorder* rec);

// -------------------------------------------------------- table builder
struct BuildStream { int n_scale, ring_head, ring_len, n_special, lpl; };
struct BuildParams {
  int n_streams, S, ring_cap, sp_cap, max_pages;
  const int* scale;          // [n_streams][S]
  const int* ring;           // [n_streams][ring_cap]
  const int* special;        // [n_streams][sp_cap]
  int* indptr;               // [n_streams+1]
  int* indices;
  int* lpl;                  // [n_streams]
  unsigned* err;
  BuildStream s[SVT_MAX_STREAMS];
};
cudaError_t launch_build_table(const BuildParams& p, cudaStream_t s, Recorder* rec);

// ------------------------------------------------------------ attention
// Per-stream slice of one attention launch.
struct StreamPlan {
  int q_off;        // first query row of the stream in q / out
  int nq;           // query rows
  int qtiles;       // ceil(nq / kTileM)
  int chunks;       // KV chunks (splits)
  int page_off;     // first entry of the stream in the visible table
  int n_pages;      // entries in the visible table
  int lpl;          // valid tokens on the last page
  int tiles;        // KV tiles: (n_pages-1)*ceil(P/TN) + ceil(lpl/TN) + ceil(extra_len/TN),
                    // TN = attn_tile_n(D)
  int item_off;     // first work item of the stream
  int extra_len;    // rows of a dense K/V segment attended after the pages (0 = none)
  int extra_off;    // first row of the stream's segment in the dense K/V arrays
};

struct AttnParams {
  int n_streams, total_items;
  int H, D, P, max_pages;    // P = tokens per pool page
  int64_t block_page_base;   // block * max_pages (page coordinate of this block's page 0)
  const int* indices;        // device visible table
  float scale_log2;          // log2(e) / sqrt(D)
  void* out;                 // [rows][H][D] cache dtype (used when chunks == 1)
  float* lse;                // [rows][H] or nullptr
  float* ws_o;               // [max_splits][ws_rows][H][D] fp32 partials
  float* ws_lse;             // [max_splits][ws_rows][H]
  int ws_rows;
  unsigned* err;
  StreamPlan s[SVT_MAX_STREAMS];
};

// Tensor-core (tcgen05 / TMEM) kernel; tensor maps are CUtensorMap (128 bytes each).
// One work item covers one 128-row query tile of one (stream, head, KV chunk).
// tmap_ke / tmap_ve map the dense K/V segments (box of TN rows); they are only
// read for streams with extra_len > 0 and may repeat another map otherwise.
int attn_items_per_stream(int H, int D, int qtiles, int chunks);
int attn_ctas_per_sm(int D);   // resident CTAs of the tensor-core kernel per SM
cudaError_t launch_attn_sm100(const AttnParams& p, const void* tmap_q, const void* tmap_kv,
                              const void* tmap_ke, const void* tmap_ve, int dtype,
                              cudaStream_t s, Recorder* rec);

// Combines split-KV partials into out / lse.
cudaError_t launch_merge(const AttnParams& p, int dtype, cudaStream_t s, Recorder* rec);

// fp32-FMA kernel (force_fp32 / fp32 pool).  Writes fp32 out and lse directly.
struct SimtStream { int q_off, nq, rblocks, page_off, n_pages, lpl, block_off, extra_len, extra_off; };
struct SimtParams {
  int n_streams, total_blocks;
  int H, D, P, max_pages;    // P = tokens per pool page
  const char* pool_block;
  const int* indices;
  const char* q;
  const char* k_extra;       // dense K/V segments [rows][H][D] (nullptr when none)
  const char* v_extra;
  float* out;
  float* lse;
  float scale;               // 1 / sqrt(D)
  unsigned* err;
  SimtStream s[SVT_MAX_STREAMS];
};
int simt_rows_per_block(int D);
cudaError_t launch_attn_simt(const SimtParams& p, int dtype, cudaStream_t s, Recorder* rec);

// Sets the thread-local message returned by svt_last_error(); returns `code`.
int report_error(int code, const char* msg);

}  // namespace svt
