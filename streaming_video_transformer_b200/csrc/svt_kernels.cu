// Memory-bound kernels of the streaming paged-attention path:
//  * append/scatter of one frame's K/V into the page pool (16-byte vectors,
//    optional fused 2-D RoPE on the patch rows of K);
//  * 2-D RoPE on the patch rows of Q;
//  * the visible-page-table builder;
//  * the split-KV merge;
//  * the fp32-FMA paged attention used for force_fp32 and fp32 pools.
//
// Pool layout: [block][max_pages][2 (K,V)][page_size][H][D]
// ("How FlashInfer's Paged KV Cache Attention Outperforms SDPA Fallback in
// Streaming Inference", Sec. Physical Memory Layout: dimension 1 separates
// keys and values).

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "svt_internal.h"

namespace svt {
namespace {

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }

// Rotates the 16-byte vectors `lo` (features i0..i0+VE-1 of a RoPE half) and
// `hi` (features i0+m/2..) by angles of position `pos`:
//   (a, b) -> (a cos - b sin, a sin + b cos),  angle_i = pos * theta^(-2i/m)
// as one fixed fp32 computation, so that the rotated keys are reproducible
// bit for bit: with c, s the fp32 table values,
//   a' = rn(rn(a c) - rn(b s)),  b' = rn(rn(a s) + rn(b c)),
// each operation rounded to nearest on its own (the _rn intrinsics keep the
// compiler from contracting a product and a sum into one fused
// multiply-add), then one rounding to the storage type.
template <typename T>
__device__ __forceinline__ void rope_pair(uint4& lo, uint4& hi, const float2* tab_row, int i0) {
  constexpr int VE = 16 / sizeof(T);
  T* a = reinterpret_cast<T*>(&lo);
  T* b = reinterpret_cast<T*>(&hi);
#pragma unroll
  for (int j = 0; j < VE; ++j) {
    const float2 cs = tab_row[i0 + j];
    const float x = to_f(a[j]), y = to_f(b[j]);
    a[j] = from_f<T>(__fsub_rn(__fmul_rn(x, cs.x), __fmul_rn(y, cs.y)));
    b[j] = from_f<T>(__fadd_rn(__fmul_rn(x, cs.y), __fmul_rn(y, cs.x)));
  }
}

// Row `row` of a frame: where it lands in the pool.  Patch rows go to
// offsets 0..P-1 of the frame's page; special rows either continue the
// stream's packed special pages or, without cross-frame retention, follow the
// patches in the frame's own page.
__device__ __forceinline__ size_t pool_offset(const AppendParams& p, int kv, int row, size_t row_bytes) {
  int page, off;
  if (row < p.ns && !p.frame_special) {
    const int n = p.sp_off0 + row;
    page = p.sp_pages[n / p.P];
    off = n % p.P;
  } else if (row < p.ns) {
    page = p.patch_page;
    off = p.P + row;
  } else {
    page = p.patch_page;
    off = row - p.ns;
  }
  return ((size_t)(page * 2 + kv) * p.page_tokens + off) * row_bytes;
}

// The K (kv = 0) or V (kv = 1) rows of one frame of one block, read from
// src, scattered into that block's pool region; grid-stride over x.
template <typename T>
__device__ __forceinline__ void append_rows(const AppendParams& p, int kv, const char* src,
                                            char* pool_block, bool mirror) {
  const size_t row_bytes = (size_t)p.H * p.D * sizeof(T);
  const int vpr = (int)(row_bytes / 16);              // vectors per row
  const int rows = p.ns + p.P;
  const long total = (long)rows * vpr;
  if (mirror && kv == 0 && blockIdx.x == 0 && threadIdx.x == 0 && p.mirror_patch) {
    *p.mirror_patch = p.patch_page;
    for (int i = 0; i < p.n_new_sp; ++i) p.mirror_special[i] = p.new_sp[i];
  }
  const bool rope = kv == 0 && p.rope_tab != nullptr;
  constexpr int VE = 16 / sizeof(T);
  const int vph = p.D / VE;                 // vectors per head
  const int half_v = vph / 4;               // vectors per RoPE quarter (m/2 features)
  const long stride = (long)gridDim.x * blockDim.x;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int row = (int)(i / vpr);
    const int vi = (int)(i % vpr);
    const size_t dst_row = pool_offset(p, kv, row, row_bytes);
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)row * row_bytes) + vi;
    uint4* d = reinterpret_cast<uint4*>(pool_block + dst_row) + vi;
    if (!rope || row < p.ns) {
      *d = __ldg(s);
      continue;
    }
    // RoPE: within a head, vectors [0, 2*half_v) form the row half, [2*half_v, 4*half_v)
    // the column half; in each half vector j < half_v pairs with j + half_v.
    const int vh = vi % vph;
    const int sect = vh / (2 * half_v);
    const int j = vh % (2 * half_v);
    if (j >= half_v) continue;              // handled by its partner
    const int patch = row - p.ns;
    const int pos = sect == 0 ? patch / p.rope_grid : patch % p.rope_grid;
    uint4 lo = __ldg(s), hi = __ldg(s + half_v);
    rope_pair<T>(lo, hi, p.rope_tab + (size_t)pos * (p.D / 4), j * VE);
    d[0] = lo;
    d[half_v] = hi;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  const int kv = blockIdx.y;
  append_rows<T>(p, kv, kv ? p.v : p.k, p.pool_block, true);
}

// Every block's append of one frame in one launch: blockIdx.z is the block.
template <typename T>
__global__ void __launch_bounds__(256) append_batch_kernel(AppendBatch b) {
  const int kv = blockIdx.y, blk = blockIdx.z;
  append_rows<T>(b.p, kv, kv ? b.v[blk] : b.k[blk], b.p.pool_block + (size_t)blk * b.block_bytes,
                 blk == 0);
}

template <typename T>
__global__ void __launch_bounds__(256) rope_q_kernel(RopeQParams p) {
  constexpr int VE = 16 / sizeof(T);
  const size_t row_bytes = (size_t)p.H * p.D * sizeof(T);
  const int vpr = (int)(row_bytes / 16);
  const int vph = p.D / VE;
  const int half_v = vph / 4;
  const long total = (long)p.rows * vpr;
  const long stride = (long)gridDim.x * blockDim.x;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int row = (int)(i / vpr);
    const int vi = (int)(i % vpr);
    const uint4* s = reinterpret_cast<const uint4*>(p.q_in + (size_t)row * row_bytes) + vi;
    uint4* d = reinterpret_cast<uint4*>(p.q_out + (size_t)row * row_bytes) + vi;
    const int local = row % p.frame_rows;
    if (local < p.ns) {
      *d = __ldg(s);
      continue;
    }
    const int vh = vi % vph;
    const int sect = vh / (2 * half_v);
    const int j = vh % (2 * half_v);
    if (j >= half_v) continue;
    const int patch = local - p.ns;
    const int pos = sect == 0 ? patch / p.rope_grid : patch % p.rope_grid;
    uint4 lo = __ldg(s), hi = __ldg(s + half_v);
    rope_pair<T>(lo, hi, p.rope_tab + (size_t)pos * (p.D / 4), j * VE);
    d[0] = lo;
    d[half_v] = hi;
  }
}

// Visible table of every stream: scale pages, window ring (oldest first),
// special pages; CSR indptr and last-page length.
__global__ void __launch_bounds__(256) build_table_kernel(BuildParams p) {
  __shared__ int off[SVT_MAX_STREAMS + 1];
  if (threadIdx.x == 0) {
    int at = 0;
    for (int i = 0; i < p.n_streams; ++i) {
      off[i] = at;
      at += p.s[i].n_scale + p.s[i].ring_len + p.s[i].n_special;
    }
    off[p.n_streams] = at;
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= p.n_streams; i += blockDim.x) p.indptr[i] = off[i];
  for (int i = threadIdx.x; i < p.n_streams; i += blockDim.x) p.lpl[i] = p.s[i].lpl;
  for (int st = 0; st < p.n_streams; ++st) {
    const BuildStream b = p.s[st];
    const int n = b.n_scale + b.ring_len + b.n_special;
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      int page;
      if (e < b.n_scale) {
        page = p.scale[st * p.S + e];
      } else if (e < b.n_scale + b.ring_len) {
        page = p.ring[st * p.ring_cap + (b.ring_head + e - b.n_scale) % p.ring_cap];
      } else {
        page = p.special[st * p.sp_cap + (e - b.n_scale - b.ring_len)];
      }
      if (page < 0 || page >= p.max_pages) {
        atomicOr(p.err, kErrPageId);
        page = 0;
      }
      p.indices[off[st] + e] = page;
    }
  }
}

// out[row,h,:] = sum_c w_c O_c / sum_c w_c,  w_c = exp(lse_c - max_c lse_c)
template <typename T>
__global__ void __launch_bounds__(128) merge_kernel(AttnParams p) {
  const int tpp = p.D / 4;                         // threads per (row, head), 4 dims each
  const int pairs_per_block = blockDim.x / tpp;
  const long pair = (long)blockIdx.x * pairs_per_block + threadIdx.x / tpp;
  const int lane = threadIdx.x % tpp;
  int total_rows = 0;
  for (int i = 0; i < p.n_streams; ++i) total_rows += p.s[i].nq;
  if (pair >= (long)total_rows * p.H) return;
  const int row = (int)(pair / p.H), h = (int)(pair % p.H);
  int chunks = 1;
  for (int i = 0; i < p.n_streams; ++i)
    if (row >= p.s[i].q_off && row < p.s[i].q_off + p.s[i].nq) chunks = p.s[i].chunks;
  if (chunks <= 1) return;                         // written directly by the attention kernel
  float mx = -INFINITY;
#pragma unroll 4
  for (int c = 0; c < chunks; ++c)
    mx = fmaxf(mx, p.ws_lse[((size_t)c * p.ws_rows + row) * p.H + h]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
#pragma unroll 4
  for (int c = 0; c < chunks; ++c) {
    const float w = __expf(p.ws_lse[((size_t)c * p.ws_rows + row) * p.H + h] - mx);
    const float4 o = reinterpret_cast<const float4*>(
        p.ws_o + (((size_t)c * p.ws_rows + row) * p.H + h) * p.D)[lane];
    acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
    den += w;
  }
  const float inv = 1.f / den;
  // four 16-bit outputs in one 8-byte store (D/4 lanes cover a row's head)
  union {
    T v[4];
    uint2 u;
  } pk;
  pk.v[0] = from_f<T>(acc.x * inv);
  pk.v[1] = from_f<T>(acc.y * inv);
  pk.v[2] = from_f<T>(acc.z * inv);
  pk.v[3] = from_f<T>(acc.w * inv);
  *reinterpret_cast<uint2*>(static_cast<T*>(p.out) + ((size_t)row * p.H + h) * p.D + lane * 4) = pk.u;
  if (p.lse && lane == 0) p.lse[(size_t)row * p.H + h] = mx + logf(den);
}

// ------------------------------------------------------ fp32 FMA attention
// TPR = D/32 threads share one query row, each owning 32 features of q and o.
// K/V tiles of KT tokens are staged in shared memory as fp32, each 32-feature
// slice padded to 33 words so that the TPR slices of one token sit in
// different banks.
constexpr int kSimtThreads = 128;
constexpr int kSimtKT = 32;

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(SimtParams p) {
  constexpr int TPR = D / 32;
  constexpr int RB = kSimtThreads / TPR;
  constexpr int SL = 33;
  __shared__ float ks[kSimtKT][TPR][SL];
  __shared__ float vs[kSimtKT][TPR][SL];
  int st = 0;
  while (st + 1 < p.n_streams && (int)blockIdx.x >= p.s[st + 1].block_off) ++st;
  const SimtStream S = p.s[st];
  const int local = blockIdx.x - S.block_off;
  const int h = local / S.rblocks;
  const int rblock = local % S.rblocks;
  const int part = threadIdx.x % TPR;
  const int r = rblock * RB + threadIdx.x / TPR;
  const bool active = r < S.nq;
  const size_t HD = (size_t)p.H * D;
  // o and l are accumulated per tile (32 terms) and the tile sums are added
  // into the running totals with Kahan compensation (oc, lc), so that streams
  // of 10^5 keys keep fp32 rounding at the level of a few ulps.
  float q[32], o[32], oc[32];
  const T* qrow = reinterpret_cast<const T*>(p.q) + (size_t)(S.q_off + (active ? r : 0)) * HD + h * D + part * 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    q[i] = active ? to_f(qrow[i]) : 0.f;
    o[i] = 0.f;
    oc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f, lc = 0.f;
  const T* pool = reinterpret_cast<const T*>(p.pool_block);
  // One tile of nt <= kSimtKT tokens whose K and V rows start at kt and vt
  // (row stride H*D): stage it, score it and fold it into (m, l, o).
  auto tile = [&](const T* kt, const T* vt, int nt) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtKT * D; e += kSimtThreads) {
      const int j = e / D, d = e % D;
      float kx = 0.f, vx = 0.f;
      if (j < nt) {
        kx = to_f(kt[(size_t)j * HD + d]);
        vx = to_f(vt[(size_t)j * HD + d]);
      }
      ks[j][d / 32][d % 32] = kx;
      vs[j][d / 32][d % 32] = vx;
    }
    __syncthreads();
    float s[kSimtKT];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kSimtKT; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc = fmaf(q[i], ks[j][part][i], acc);
#pragma unroll
      for (int w = 1; w < TPR; w <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
      s[j] = j < nt ? acc * p.scale : -INFINITY;
      tmax = fmaxf(tmax, s[j]);
    }
    const float mnew = fmaxf(m, tmax);
    const float alpha = expf(m - mnew);   // m = -inf on the first tile -> 0
    m = mnew;
    float ot[32], lt = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) ot[i] = 0.f;
#pragma unroll
    for (int j = 0; j < kSimtKT; ++j) {
      const float pj = expf(s[j] - m);
      lt += pj;
#pragma unroll
      for (int i = 0; i < 32; ++i) ot[i] = fmaf(pj, vs[j][part][i], ot[i]);
    }
    {
      const float lr = __fmul_rn(l, alpha), lcr = __fmul_rn(lc, alpha);
      const float y = __fsub_rn(lt, lcr);
      const float tt = __fadd_rn(lr, y);
      lc = __fsub_rn(__fsub_rn(tt, lr), y);
      l = tt;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float orr = __fmul_rn(o[i], alpha), ocr = __fmul_rn(oc[i], alpha);
      const float y = __fsub_rn(ot[i], ocr);
      const float tt = __fadd_rn(orr, y);
      oc[i] = __fsub_rn(__fsub_rn(tt, orr), y);
      o[i] = tt;
    }
  };
  for (int pp = 0; pp < S.n_pages; ++pp) {
    int page = p.indices[S.page_off + pp];
    if (page < 0 || page >= p.max_pages) {
      if (threadIdx.x == 0) atomicOr(p.err, kErrPageId);
      page = 0;
    }
    const int valid = pp == S.n_pages - 1 ? S.lpl : p.P;
    const T* kpage = pool + (size_t)page * 2 * p.P * HD + h * D;
    const T* vpage = kpage + (size_t)p.P * HD;
    for (int t0 = 0; t0 < valid; t0 += kSimtKT)
      tile(kpage + (size_t)t0 * HD, vpage + (size_t)t0 * HD, min(kSimtKT, valid - t0));
  }
  // The stream's dense K/V segment (a frame attended without being stored).
  if (S.extra_len > 0) {
    const T* ke = reinterpret_cast<const T*>(p.k_extra) + (size_t)S.extra_off * HD + h * D;
    const T* ve = reinterpret_cast<const T*>(p.v_extra) + (size_t)S.extra_off * HD + h * D;
    for (int t0 = 0; t0 < S.extra_len; t0 += kSimtKT)
      tile(ke + (size_t)t0 * HD, ve + (size_t)t0 * HD, min(kSimtKT, S.extra_len - t0));
  }
  if (!active) return;
  const float inv = 1.f / l;
  float* orow = p.out + (size_t)(S.q_off + r) * HD + h * D + part * 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) orow[i] = o[i] * inv;
  if (p.lse && part == 0) p.lse[(size_t)(S.q_off + r) * p.H + h] = m + logf(l);
}

template <typename T>
cudaError_t launch_simt_t(const SimtParams& p, cudaStream_t s, Recorder* rec) {
  if (p.total_blocks == 0) return cudaSuccess;
  switch (p.D) {
    case 32: return dispatch(rec, attn_simt_kernel<T, 32>, p.total_blocks, kSimtThreads, 0, s, p);
    case 64: return dispatch(rec, attn_simt_kernel<T, 64>, p.total_blocks, kSimtThreads, 0, s, p);
    case 128: return dispatch(rec, attn_simt_kernel<T, 128>, p.total_blocks, kSimtThreads, 0, s, p);
    default: return cudaErrorInvalidValue;
  }
}

int grid_for(long work, int threads) {
  long b = (work + threads - 1) / threads;
  return (int)std::min<long>(std::max<long>(b, 1), 148L * 16);
}

}  // namespace

int simt_rows_per_block(int D) { return kSimtThreads / (D / 32); }

cudaError_t launch_append(const AppendParams& p, int dtype, cudaStream_t s, Recorder* rec) {
  const long vecs = (long)(p.ns + p.P) * p.H * p.D * p.elem / 16;
  dim3 grid(grid_for(vecs, 256), 2);
  switch (dtype) {
    case SVT_BF16: return dispatch(rec, append_kernel<__nv_bfloat16>, grid, 256, 0, s, p);
    case SVT_FP16: return dispatch(rec, append_kernel<__half>, grid, 256, 0, s, p);
    default: return dispatch(rec, append_kernel<float>, grid, 256, 0, s, p);
  }
}

cudaError_t launch_append_batch(const AppendBatch& b, int dtype, cudaStream_t s, Recorder* rec) {
  const AppendParams& p = b.p;
  const long vecs = (long)(p.ns + p.P) * p.H * p.D * p.elem / 16;
  dim3 grid(std::max(1, grid_for(vecs, 256) / std::max(1, b.n_blocks / 4)), 2, b.n_blocks);
  switch (dtype) {
    case SVT_BF16: return dispatch(rec, append_batch_kernel<__nv_bfloat16>, grid, 256, 0, s, b);
    case SVT_FP16: return dispatch(rec, append_batch_kernel<__half>, grid, 256, 0, s, b);
    default: return dispatch(rec, append_batch_kernel<float>, grid, 256, 0, s, b);
  }
}

cudaError_t launch_rope_q(const RopeQParams& p, int dtype, cudaStream_t s, Recorder* rec) {
  const long vecs = (long)p.rows * p.H * p.D * p.elem / 16;
  const int grid = grid_for(vecs, 256);
  switch (dtype) {
    case SVT_BF16: return dispatch(rec, rope_q_kernel<__nv_bfloat16>, grid, 256, 0, s, p);
    case SVT_FP16: return dispatch(rec, rope_q_kernel<__half>, grid, 256, 0, s, p);
    default: return dispatch(rec, rope_q_kernel<float>, grid, 256, 0, s, p);
  }
}

cudaError_t launch_build_table(const BuildParams& p, cudaStream_t s, Recorder* rec) {
  return dispatch(rec, build_table_kernel, 1, 256, 0, s, p);
}

cudaError_t launch_merge(const AttnParams& p, int dtype, cudaStream_t s, Recorder* rec) {
  int rows = 0;
  for (int i = 0; i < p.n_streams; ++i) rows += p.s[i].nq;
  const int tpp = p.D / 4;
  const int pairs_per_block = 128 / tpp;
  const long pairs = (long)rows * p.H;
  const int grid = (int)((pairs + pairs_per_block - 1) / pairs_per_block);
  if (grid == 0) return cudaSuccess;
  if (dtype == SVT_BF16) return dispatch(rec, merge_kernel<__nv_bfloat16>, grid, 128, 0, s, p);
  return dispatch(rec, merge_kernel<__half>, grid, 128, 0, s, p);
}

cudaError_t launch_attn_simt(const SimtParams& p, int dtype, cudaStream_t s, Recorder* rec) {
  switch (dtype) {
    case SVT_BF16: return launch_simt_t<__nv_bfloat16>(p, s, rec);
    case SVT_FP16: return launch_simt_t<__half>(p, s, rec);
    default: return launch_simt_t<float>(p, s, rec);
  }
}

}  // namespace svt
