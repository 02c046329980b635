// Paged attention on the sm_100a tensor cores (tcgen05 MMA, TMEM accumulators,
// TMA page gathers).
//
// What it computes ("How Paged KV Cache Attention Enables ~20 FPS Streaming
// Inference in LingBot-Map", Sec. FlashInfer Paged-Kernel Integration and
// Sec. Step-by-Step Streaming Inference, step 4; "How the Paged KV Cache
// Attention Mechanism Enables Long Sequence Inference in LingBot-Map",
// Sec. FlashInfer Kernel Execution): for one frame's queries, softmax over
// every visible token of the stream -- the pages listed by the visible page
// table, each full except the last (last_page_len valid tokens) -- with no
// causal mask, read straight from the page pool.
//
// Work item = (stream, head, pair of 128-row query tiles, KV chunk); one CTA
// per item, 320 threads:
//   warp 8      TMA producer: both Q tiles once, then K and V tiles of 128
//               tokens gathered page by page through the visible table (a
//               page is ceil(page_size/128) tiles; rows past the page end are
//               zero-filled by TMA and masked).
//   warp 9      MMA issuer (one thread) and TMEM owner.  Per KV tile j:
//                 S0_j = Q0 K_j^T, S1_j = Q1 K_j^T       (SS MMA into TMEM)
//                 O0 += P0_j V_j,  O1 += P1_j V_j        (TS MMA, P from TMEM)
//               in the order S0_0 S1_0 | PV0_0 S0_1 PV1_0 S1_1 | PV0_1 ...
//   warps 0-3   softmax of query tile 0, warps 4-7 of query tile 1: thread r
//               owns row r (TMEM lane r), reads S, keeps the running max and
//               sum in the log2 domain, rescales O lazily (only when the max
//               grows by more than 2^8), writes P as 16-bit pairs over the
//               first half of S's columns; then the epilogue (O / l, LSE).
// The two softmax warpgroups ping-pong: one works on its S while the tensor
// cores run the other tile's P.V and next S.  K/V tiles are loaded once for
// both query tiles.  Split-KV chunks write fp32 partials and LSE; a merge
// kernel combines them.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_primitives.cuh"
#include "svt_internal.h"

#ifndef SVT_EXP_MODE
#define SVT_EXP_MODE 0   // 0: fp32 MUFU exp2; 1: packed f16x2 MUFU exp2 (two per instruction)
#endif

namespace svt {
namespace {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr float kRescaleThreshold = 8.0f;          // log2 units

template <int D>
struct Cfg {
  static constexpr int kRegions = D / 64;                      // 64-feature swizzle columns
  static constexpr uint32_t kTileBytes = kTileN * D * 2;       // one K, V or Q tile
  static constexpr uint32_t kRegionBytes = kTileN * 128;       // 128 rows x 128 bytes
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr uint32_t kQOff = 0;                          // two Q tiles
  static constexpr uint32_t kKOff = 2 * kTileBytes;
  static constexpr uint32_t kVOff = kKOff + kStages * kTileBytes;
  static constexpr uint32_t kBarOff = kVOff + kStages * kTileBytes;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], o_done[2], drain
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 2 + 1;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;   // + alignment slack
  static constexpr uint32_t kTmemS = 0;        // S of tile x at column 128 x
  static constexpr uint32_t kTmemO = 256;      // O of tile x at column 256 + D x
};

struct Item {
  int st, head, qpair, chunk, t_begin, n_tiles;
  bool two;   // the pair's second query tile holds rows of this stream
};

__device__ __forceinline__ Item decode_item(const AttnParams& p) {
  Item it;
  int st = 0;
  while (st + 1 < p.n_streams && (int)blockIdx.x >= p.s[st + 1].item_off) ++st;
  const StreamPlan& sp = p.s[st];
  const int qpairs = (sp.qtiles + 1) / 2;
  const int local = blockIdx.x - sp.item_off;
  it.st = st;
  it.qpair = local % qpairs;
  const int rest = local / qpairs;
  it.chunk = rest % sp.chunks;
  it.head = rest / sp.chunks;
  it.two = 2 * it.qpair + 1 < sp.qtiles;
  const int t0 = (int)((int64_t)it.chunk * sp.tiles / sp.chunks);
  const int t1 = (int)((int64_t)(it.chunk + 1) * sp.tiles / sp.chunks);
  it.t_begin = t0;
  it.n_tiles = t1 - t0;
  return it;
}

// Tile g of a stream's KV sequence -> (position in the visible table, tile in page, valid rows).
__device__ __forceinline__ void tile_coords(const StreamPlan& sp, int P, int g, int& page_pos,
                                            int& t, int& valid) {
  const int tpp = (P + kTileN - 1) / kTileN;
  const int full = (sp.n_pages - 1) * tpp;
  int page_tokens;
  if (g < full) {
    page_pos = g / tpp;
    t = g % tpp;
    page_tokens = P;
  } else {
    page_pos = sp.n_pages - 1;
    t = g - full;
    page_tokens = sp.lpl;
  }
  valid = min(kTileN, page_tokens - t * kTileN);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h2);
  } else {
    __half2 h2 = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h2);
  }
}

template <int D, bool BF16>
__global__ void __maxnreg__(192)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_kv,
                      const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sK = base + C::kKOff;
  const uint32_t sV = base + C::kVOff;
  const uint32_t bars = base + C::kBarOff;
  const uint32_t q_full = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + C::kStages + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * C::kStages + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 3 * C::kStages + s); };
  auto s_full = [&](int x) { return bars + 8u * (1 + 4 * C::kStages + x); };
  auto p_full = [&](int x) { return bars + 8u * (3 + 4 * C::kStages + x); };
  auto o_done = [&](int x) { return bars + 8u * (5 + 4 * C::kStages + x); };
  const uint32_t drain = bars + 8u * (7 + 4 * C::kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const Item it = decode_item(p);
  const StreamPlan& sp = p.s[it.st];
  const int n = it.n_tiles;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), 128);
      mbar_init(o_done(x), 1);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 9) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(p.err, kErrWaitLimit);
  };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_kv);
      const int q_row0 = sp.q_off + 2 * it.qpair * kTileM;
      mbar_arrive_expect_tx(q_full, (it.two ? 2 : 1) * C::kTileBytes);
      for (int x = 0; x < (it.two ? 2 : 1); ++x)
        for (int r = 0; r < C::kRegions; ++r)
          tma_load_3d(sQ + x * C::kTileBytes + r * C::kRegionBytes, &tmap_q, q_full, r * 64,
                      it.head, q_row0 + x * kTileM);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        int page_pos, t, valid;
        tile_coords(sp, p.P, it.t_begin + j, page_pos, t, valid);
        int page = p.indices[sp.page_off + page_pos];
        if (page < 0 || page >= p.max_pages) {
          atomicOr(p.err, kErrPageId);
          page = 0;
        }
        const int c4 = (int)(p.block_page_base + page);
        const int s = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!mbar_wait(k_empty(s), ph ^ 1, abort_flag, kWaitLimitNs)) { fail(); break; }
        mbar_arrive_expect_tx(k_full(s), C::kTileBytes);
        for (int r = 0; r < C::kRegions; ++r)
          tma_load_5d(sK + s * C::kTileBytes + r * C::kRegionBytes, &tmap_kv, k_full(s), r * 64,
                      it.head, t * kTileN, 0, c4);
        issued = j + 1;
        if (!mbar_wait(v_empty(s), ph ^ 1, abort_flag, kWaitLimitNs)) { fail(); break; }
        mbar_arrive_expect_tx(v_full(s), C::kTileBytes);
        for (int r = 0; r < C::kRegions; ++r)
          tma_load_5d(sV + s * C::kTileBytes + r * C::kRegionBytes, &tmap_kv, v_full(s), r * 64,
                      it.head, t * kTileN, 1, c4);
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        mbar_wait(q_full, 0, nullptr, kWaitLimitNs);
        for (int j = max(0, issued - C::kStages); j < issued; ++j) {
          const int s = j % C::kStages;
          const uint32_t ph = (j / C::kStages) & 1;
          mbar_wait(k_full(s), ph, nullptr, kWaitLimitNs);
          mbar_wait(v_full(s), ph, nullptr, kWaitLimitNs);
        }
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(kTileM, kTileN, BF16, false);
      constexpr uint32_t idO = idesc_f16(kTileM, D, BF16, true);
      const int nx = it.two ? 2 : 1;
      bool ok = mbar_wait(q_full, 0, abort_flag, kWaitLimitNs);
      tc_fence_after();
      // S_x = Q_x K_j^T into tile x's S columns.
      auto issue_s = [&](int x, int j) {
        const uint32_t kb = sK + (j % C::kStages) * C::kTileBytes;
        const uint32_t qb = sQ + x * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kRegionBytes + (kk % 4) * 32;
          mma_ss(tmem + C::kTmemS + 128 * x, desc_sw128(qb + off, 16, 1024),
                 desc_sw128(kb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full(x));
      };
      // O_x += P_x V_j with P_x read from tile x's S columns.
      auto issue_pv = [&](int x, int j) {
        const uint32_t vb = sV + (j % C::kStages) * C::kTileBytes;
        const uint32_t a = tmem + C::kTmemS + 128 * x;
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)
          mma_ts(tmem + C::kTmemO + D * x, a + kk * 8,
                 desc_sw128(vb + kk * 2048, C::kRegionBytes, 1024), idO,
                 (j > 0 || kk > 0) ? 1u : 0u);
      };
      if (ok && n > 0) {
        ok = mbar_wait(k_full(0), 0, abort_flag, kWaitLimitNs);
        if (ok) {
          tc_fence_after();
          for (int x = 0; x < nx; ++x) issue_s(x, 0);
          mma_commit(k_empty(0));
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        const int s = j % C::kStages;
        const int s1 = (j + 1) % C::kStages;
        const bool more = j + 1 < n;
        for (int x = 0; x < nx && ok; ++x) {
          if (!(ok = mbar_wait(p_full(x), j & 1, abort_flag, kWaitLimitNs))) break;
          if (x == 0 && !(ok = mbar_wait(v_full(s), (j / C::kStages) & 1, abort_flag,
                                         kWaitLimitNs)))
            break;
          tc_fence_after();
          issue_pv(x, j);
          if (!more) mma_commit(o_done(x));
          if (x == nx - 1) mma_commit(v_empty(s));
          if (more) {
            if (x == 0 && !(ok = mbar_wait(k_full(s1), ((j + 1) / C::kStages) & 1, abort_flag,
                                           kWaitLimitNs)))
              break;
            tc_fence_after();
            issue_s(x, j + 1);
            if (x == nx - 1) mma_commit(k_empty(s1));
          }
        }
      }
      if (!ok) fail();
      // Drain: every MMA issued above has completed once `drain` flips.
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kWaitLimitNs);
    }
  } else if (warp < 4 || it.two) {
    // ------------------------------------------------------ softmax warps
    // Warps 4x..4x+3 own query tile x.  Every tcgen05.ld/st below runs on all
    // 32 lanes of a warp (the branches around them are warp-uniform).  S_x of
    // tile j is issued after P_x.V of tile j-1, so once S_x has arrived the
    // tile's O is quiescent and may be rescaled without a further wait.
    const int x = warp / 4;
    const int row = threadIdx.x % 128;                         // TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t sb = lane_addr + C::kTmemS + 128 * x;
    const uint32_t ob = lane_addr + C::kTmemO + D * x;
    const float sl2 = p.scale_log2;
    constexpr unsigned kAll = 0xffffffffu;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(kAll, mbar_wait(s_full(x), j & 1, abort_flag, kWaitLimitNs));
      if (!ok) break;
      tc_fence_after();
      int page_pos, t, valid;
      tile_coords(sp, p.P, it.t_begin + j, page_pos, t, valid);
      float s[128];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(sb, r0);
        tmem_ld32(sb + 32, r1);
        tmem_ld32(sb + 64, r2);
        tmem_ld32(sb + 96, r3);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = __uint_as_float(r0[i]);
          s[32 + i] = __uint_as_float(r1[i]);
          s[64 + i] = __uint_as_float(r2[i]);
          s[96 + i] = __uint_as_float(r3[i]);
        }
      }
      if (valid < kTileN) {
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = i < valid ? s[i] : -INFINITY;
      }
      float mx;
      {
        float mm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mm[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
        for (int i = 8; i < 64; ++i) mm[i % 8] = fmax3(mm[i % 8], s[2 * i], s[2 * i + 1]);
        mx = fmax3(fmax3(mm[0], mm[1], mm[2]), fmax3(mm[3], mm[4], mm[5]), fmaxf(mm[6], mm[7]));
      }
      mx *= sl2;
      // New running max.  The O rescale it may need is done after P is
      // written (S registers are dead by then) and before P_x is released.
      bool rescale = false;
      float alpha = 1.f;
      if (j == 0) {
        m = mx;
      } else if (__any_sync(kAll, mx > m + kRescaleThreshold)) {
        const float mnew = fmaxf(m, mx);
        alpha = ex2(m - mnew);
        l *= alpha;
        m = mnew;
        rescale = true;
      }
      const float nm = -m;
      float la[4] = {0.f, 0.f, 0.f, 0.f}, lb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1, p0, p1;
          ffma2(x0, x1, s[32 * c + 2 * i], s[32 * c + 2 * i + 1], sl2, sl2, nm, nm);
#if SVT_EXP_MODE == 1
          ex2_h2(p0, p1, x0, x1);
#else
          p0 = ex2(x0);
          p1 = ex2(x1);
#endif
          fadd2(la[i % 4], lb[i % 4], la[i % 4], lb[i % 4], p0, p1);
          pk[i] = pack2<BF16>(p0, p1);
        }
        tmem_st16(sb + 16 * c, pk);
      }
      l += (la[0] + lb[0]) + (la[1] + lb[1]) + (la[2] + lb[2]) + (la[3] + lb[3]);
      if (rescale) {
        // O holds the sum over earlier tiles scaled by 2^-m_old: move it to 2^-m.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(ob + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(ob + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(x));
    }
    if (ok && n > 0) ok = __all_sync(kAll, mbar_wait(o_done(x), 0, abort_flag, kWaitLimitNs));
    if (!ok) fail();
    tc_fence_after();
    if (ok && n > 0) {
      const int r = (2 * it.qpair + x) * kTileM + row;
      const bool store = r < sp.nq;
      const float inv = 1.f / l;
      const int grow = sp.q_off + (store ? r : 0);
      const float lse = (m + __log2f(l)) * 0.69314718055994531f;
      if (sp.chunks == 1) {
        T* orow = static_cast<T*>(p.out) + ((size_t)grow * p.H + it.head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(ob + c * 32, o);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if (store && p.lse) p.lse[(size_t)grow * p.H + it.head] = lse;
      } else {
        const size_t wrow = ((size_t)it.chunk * p.ws_rows + grow) * p.H + it.head;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + wrow * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(ob + c * 32, o);
          tmem_wait_ld();
          if (store) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[c * 8 + v] = make_float4(__uint_as_float(o[4 * v]) * inv,
                                           __uint_as_float(o[4 * v + 1]) * inv,
                                           __uint_as_float(o[4 * v + 2]) * inv,
                                           __uint_as_float(o[4 * v + 3]) * inv);
          }
        }
        if (store) p.ws_lse[wrow] = lse;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool BF16>
cudaError_t launch_t(const AttnParams& p, const void* tq, const void* tkv, cudaStream_t s) {
  using C = Cfg<D>;
  auto kern = attn_sm100_kernel<D, BF16>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  CUtensorMap mq, mkv;
  memcpy(&mq, tq, sizeof(mq));
  memcpy(&mkv, tkv, sizeof(mkv));
  kern<<<p.total_items, kThreads, C::kSmemBytes, s>>>(mq, mkv, p);
  return cudaGetLastError();
}

}  // namespace

int attn_items_per_stream(int H, int qtiles, int chunks) { return H * ((qtiles + 1) / 2) * chunks; }

cudaError_t launch_attn_sm100(const AttnParams& p, const void* tmap_q, const void* tmap_kv,
                              int dtype, cudaStream_t s) {
  if (p.total_items == 0) return cudaSuccess;
  const bool bf16 = dtype == SVT_BF16;
  if (p.D == 64) return bf16 ? launch_t<64, true>(p, tmap_q, tmap_kv, s)
                             : launch_t<64, false>(p, tmap_q, tmap_kv, s);
  if (p.D == 128) return bf16 ? launch_t<128, true>(p, tmap_q, tmap_kv, s)
                              : launch_t<128, false>(p, tmap_q, tmap_kv, s);
  return cudaErrorInvalidValue;
}

}  // namespace svt
