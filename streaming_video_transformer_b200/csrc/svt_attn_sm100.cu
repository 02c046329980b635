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
// Work item = (stream, head, 128-row query tile, KV chunk); one CTA per item.
// KV tiles hold TN tokens (128 at D = 64, 64 at D = 128), so a CTA takes 256
// TMEM columns and under half an SM's shared memory and two CTAs share an SM.
// D = 128 runs 192 threads; D = 64 runs 256 (warps 6-7 only hand their
// registers to the softmax warpgroup):
//   warp 4      TMA producer: the Q tile once, then K and V tiles of TN
//               tokens gathered page by page through the visible table (a
//               page is ceil(page_size/TN) tiles; rows past the page end are
//               zero-filled by TMA and masked).
//   warp 5      MMA issuer (one thread) and TMEM owner:
//                 S_j = Q K_j^T   (SS MMA, fp32 into TMEM columns 0..TN-1)
//                 O  += P_j V_j   (TS MMA: P_j from TMEM columns TN..3TN/2-1)
//               S_{j+1} is issued as soon as the softmax has read S_j, so the
//               tensor cores compute it while the softmax exponentiates S_j.
//   warps 0-3   softmax: thread r owns query row r (TMEM lane r): reads S_j
//               and releases it, exponentiates in the log2 domain against the
//               running maximum of the earlier tiles (no reduction over the
//               tile first), writes P_j as 16-bit pairs once P_{j-1}.V_{j-1}
//               has completed (which also leaves O quiescent for a rescale),
//               and recomputes the tile against its exact maximum only when
//               the row sum of P_j exceeds 2^8 (always on the first tile).
// At D = 64 a tile needs twice as many exponential-unit cycles as tensor
// cycles (one exp per 256 MMA flops), but the measured limit is the latency of
// each CTA's S -> softmax -> P -> P.V chain; the two CTAs on an SM overlap
// their chains.
// Split-KV chunks write fp32 partials and LSE; a merge kernel combines them.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_primitives.cuh"
#include "svt_internal.h"

namespace svt {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
// D = 64 launches 256 threads (two warpgroups) with 128 registers each and
// moves registers from the producer/MMA warpgroup (warps 4-7, down to 64) to
// the softmax warpgroup (warps 0-3, up to 192): 128 x 64 + 128 x 192 = 256 x
// 128.  The build checks that the kernel's launch register count is 128; a
// smaller count would leave the increase waiting for registers forever.
constexpr int kSplitThreads = 256;
constexpr int threads_for(int D) { return D == 64 ? kSplitThreads : kThreads; }
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
// A tile's P row is accepted while its sum stays at or below this bound, so
// that every P value is at most 2^8 (within fp16's range for the P.V MMA).
constexpr float kRowSumBound = 256.0f;

template <int D>
struct Cfg {
  static constexpr int TN = attn_tile_n(D);                    // KV tokens per tile
  static constexpr int kRegions = D / 64;                      // 64-feature swizzle columns
  static constexpr uint32_t kQBytes = kTileM * D * 2;          // the Q tile
  static constexpr uint32_t kQRegionBytes = kTileM * 128;      // 128 rows x 128 bytes
  static constexpr uint32_t kKVBytes = TN * D * 2;             // one K or V tile
  static constexpr uint32_t kKVRegionBytes = TN * 128;         // TN rows x 128 bytes
  // K and V rings; a CTA stays under half an SM's shared memory.
  static constexpr int kKStages = D == 64 ? 3 : 2;
  static constexpr int kVStages = 2;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQBytes;
  static constexpr uint32_t kVOff = kKOff + kKStages * kKVBytes;
  static constexpr uint32_t kBarOff = kVOff + kVStages * kKVBytes;
  // q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full, s_free, p_full, o_done,
  // drain
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 5;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;   // + alignment slack
  // TMEM, 256 columns so that two CTAs share an SM: S (TN fp32 columns) at
  // 0, P (TN/2 columns of 16-bit pairs) at TN, O (D fp32 columns) at 256 - D.
  // D = 64: S 0..127, P 128..191, O 192..255; D = 128: S 0..63, P 64..95,
  // O 128..255.
  static constexpr uint32_t kTmemS = 0;
  static constexpr uint32_t kTmemP = TN;
  static constexpr uint32_t kTmemO = 256 - D;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(kTmemP + TN / 2 <= kTmemO, "TMEM layout overlaps");
};

struct Item {
  int st, head, qtile, chunk, t_begin, n_tiles;
};

__device__ __forceinline__ Item decode_item(const AttnParams& p) {
  Item it;
  int st = 0;
  while (st + 1 < p.n_streams && (int)blockIdx.x >= p.s[st + 1].item_off) ++st;
  const StreamPlan& sp = p.s[st];
  const int local = blockIdx.x - sp.item_off;
  it.st = st;
  it.qtile = local % sp.qtiles;
  const int rest = local / sp.qtiles;
  it.chunk = rest % sp.chunks;
  it.head = rest / sp.chunks;
  const int t0 = (int)((int64_t)it.chunk * sp.tiles / sp.chunks);
  const int t1 = (int)((int64_t)(it.chunk + 1) * sp.tiles / sp.chunks);
  it.t_begin = t0;
  it.n_tiles = t1 - t0;
  return it;
}

// Tile g of a stream's KV sequence -> (position in the visible table, tile in page, valid rows).
template <int TN>
__device__ __forceinline__ void tile_coords(const StreamPlan& sp, int P, int g, int& page_pos,
                                            int& t, int& valid) {
  const int tpp = (P + TN - 1) / TN;
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
  valid = min(TN, page_tokens - t * TN);
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
__global__ void __launch_bounds__(threads_for(D), 2)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_kv,
                      const __grid_constant__ CUtensorMap tmap_ke,
                      const __grid_constant__ CUtensorMap tmap_ve,
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
  constexpr int KS = C::kKStages, VS = C::kVStages, TN = C::TN;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + KS + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * KS + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 2 * KS + VS + s); };
  const uint32_t s_full = bars + 8u * (1 + 2 * KS + 2 * VS);
  const uint32_t s_free = s_full + 8u;
  const uint32_t p_full = s_full + 16u;
  const uint32_t o_done = s_full + 24u;
  const uint32_t drain = s_full + 32u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const Item it = decode_item(p);
  const StreamPlan& sp = p.s[it.st];
  const int n = it.n_tiles;
  // Tiles [0, page_tiles) of the stream come from the page table, the rest
  // from its dense K/V segment (a frame attended without being stored).
  const int page_tiles = sp.tiles - (sp.extra_len + TN - 1) / TN;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
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

  if (warp >= 4) {
  if constexpr (D == 64) asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_kv);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
      for (int r = 0; r < C::kRegions; ++r)
        tma_load_3d(sQ + r * C::kQRegionBytes, &tmap_q, q_full, r * 64, it.head,
                    sp.q_off + it.qtile * kTileM);
      if (sp.extra_len > 0) {
        tma_prefetch_desc(&tmap_ke);
        tma_prefetch_desc(&tmap_ve);
      }
      int issued = 0, vissued = 0;
      for (int j = 0; j < n; ++j) {
        const int g = it.t_begin + j;
        int page_pos = 0, t = 0, valid, c4 = 0, erow = 0;
        const bool extra = g >= page_tiles;
        if (extra) {
          erow = sp.extra_off + (g - page_tiles) * TN;   // rows past the segment are masked
        } else {
          tile_coords<TN>(sp, p.P, g, page_pos, t, valid);
          int page = p.indices[sp.page_off + page_pos];
          if (page < 0 || page >= p.max_pages) {
            atomicOr(p.err, kErrPageId);
            page = 0;
          }
          c4 = (int)(p.block_page_base + page);
        }
        const int sk = j % KS, sv = j % VS;
        if (!mbar_wait(k_empty(sk), ((j / KS) & 1) ^ 1, abort_flag, kWaitLimitNs)) { fail(); break; }
        mbar_arrive_expect_tx(k_full(sk), C::kKVBytes);
        for (int r = 0; r < C::kRegions; ++r) {
          const uint32_t dst = sK + sk * C::kKVBytes + r * C::kKVRegionBytes;
          if (extra)
            tma_load_3d(dst, &tmap_ke, k_full(sk), r * 64, it.head, erow);
          else
            tma_load_5d(dst, &tmap_kv, k_full(sk), r * 64, it.head, t * TN, 0, c4);
        }
        issued = j + 1;
        if (!mbar_wait(v_empty(sv), ((j / VS) & 1) ^ 1, abort_flag, kWaitLimitNs)) { fail(); break; }
        mbar_arrive_expect_tx(v_full(sv), C::kKVBytes);
        for (int r = 0; r < C::kRegions; ++r) {
          const uint32_t dst = sV + sv * C::kKVBytes + r * C::kKVRegionBytes;
          if (extra)
            tma_load_3d(dst, &tmap_ve, v_full(sv), r * 64, it.head, erow);
          else
            tma_load_5d(dst, &tmap_kv, v_full(sv), r * 64, it.head, t * TN, 1, c4);
        }
        vissued = j + 1;
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        mbar_wait(q_full, 0, nullptr, kWaitLimitNs);
        for (int j = max(0, issued - KS); j < issued; ++j)
          mbar_wait(k_full(j % KS), (j / KS) & 1, nullptr, kWaitLimitNs);
        for (int j = max(0, vissued - VS); j < vissued; ++j)
          mbar_wait(v_full(j % VS), (j / VS) & 1, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(kTileM, TN, BF16, false);
      constexpr uint32_t idO = idesc_f16(kTileM, D, BF16, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, kWaitLimitNs);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int s = j % KS;
        if (!mbar_wait(k_full(s), (j / KS) & 1, abort_flag, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t kb = sK + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t in_row = (kk % 4) * 32;
          mma_ss(tmem + C::kTmemS, desc_sw128(sQ + (kk / 4) * C::kQRegionBytes + in_row, 16, 1024),
                 desc_sw128(kb + (kk / 4) * C::kKVRegionBytes + in_row, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(k_empty(s));
        mma_commit(s_full);
        return true;
      };
      if (ok && n > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          // S_{j+1} overwrites S_j once the softmax has read it.
          if (!(ok = mbar_wait(s_free, j & 1, abort_flag, kWaitLimitNs))) break;
          tc_fence_after();
          if (!(ok = issue_s(j + 1))) break;
        }
        const int s = j % VS;
        if (!(ok = mbar_wait(p_full, j & 1, abort_flag, kWaitLimitNs))) break;
        if (!(ok = mbar_wait(v_full(s), (j / VS) & 1, abort_flag, kWaitLimitNs))) break;
        tc_fence_after();
        const uint32_t vb = sV + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk)
          mma_ts(tmem + C::kTmemO, tmem + C::kTmemP + kk * 8,
                 desc_sw128(vb + kk * 2048, C::kKVRegionBytes, 1024), idO,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(v_empty(s));
        mma_commit(o_done);
      }
      if (!ok) fail();
      // Drain: every MMA issued above has completed once `drain` flips.
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kWaitLimitNs);
    }
  }
  } else {
    if constexpr (D == 64) asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    // ------------------------------------------------------ softmax warps
    // Every tcgen05.ld/st runs on all 32 lanes of a warp (the branches around
    // them are warp-uniform).
    const int row = threadIdx.x;                               // TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t sb = lane_addr + C::kTmemS;
    const uint32_t pb = lane_addr + C::kTmemP;
    const uint32_t ob = lane_addr + C::kTmemO;
    const float sl2 = p.scale_log2;
    constexpr unsigned kAll = 0xffffffffu;
    // Running maximum m (log2 units): very negative but finite at the start,
    // so that the first tile's exponentials overflow to +inf, its row-sum
    // test fails and it is computed against its exact maximum; masked (-inf)
    // scores still give 0.
    float m = -1e30f, l = 0.f;
    bool ok = true;
    // Position of the current tile in the visible table, advanced by one
    // tile per iteration (no divisions on the per-tile path).
    const int tpp = (p.P + TN - 1) / TN;
    const int last_page = sp.n_pages - 1, lpl = sp.lpl, P = p.P;
    int page_pos, t, valid;
    tile_coords<TN>(sp, P, it.t_begin, page_pos, t, valid);
    for (int j = 0; j < n && ok; ++j) {
      if (it.t_begin + j < page_tiles) {
        valid = min(TN, (page_pos < last_page ? P : lpl) - t * TN);
        if (++t == tpp && page_pos < last_page) {
          t = 0;
          ++page_pos;
        }
      } else {
        valid = min(TN, sp.extra_len - (it.t_begin + j - page_tiles) * TN);
      }
      ok = __all_sync(kAll, mbar_wait(s_full, j & 1, abort_flag, kWaitLimitNs));
      if (!ok) break;
      tc_fence_after();
      constexpr int NC = TN / 32;                     // 32-column chunks per tile
      float s[TN];
      {
        uint32_t r[NC][32];
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(sb + 32 * c, r[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(s_free);
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[c][i]);
      }
      if (valid < TN) {
#pragma unroll
        for (int i = 0; i < TN; ++i) s[i] = i < valid ? s[i] : -INFINITY;
      }
      // The exponentials are taken against the running maximum m of the
      // earlier tiles, without a reduction over this tile first.  P values
      // are non-negative, so the row sum bounds each of them: while it stays
      // at or below kRowSumBound, P, l and O are consistent with m and the
      // tile stands as computed (online softmax is exact for any m; the
      // bound only keeps P in range).  Otherwise (the first tile, or a score
      // more than one log2 unit above m) the tile's maximum is reduced, m is
      // raised to it, and the tile is recomputed.
      float la[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const float nm = -m;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint32_t pk[16];
          if (c == NC - 1 && valid <= 32 * (NC - 1)) {
            // The last chunk lies wholly past the tile's valid rows (the
            // tail tile of a page): P = 0 without exponentiating -inf.
            // Only the last chunk is tested, so no branch separates the
            // exponentials of consecutive chunks.
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = ex2(fmaf(s[32 * c + 2 * i], sl2, nm));
              const float p1 = ex2(fmaf(s[32 * c + 2 * i + 1], sl2, nm));
              la[i % 4] += p0 + p1;
              pk[i] = pack2<BF16>(p0, p1);
            }
          }
          // P_{j-1}.V_{j-1} must have read the P columns (and finished
          // updating O) before P_j is written and O rescaled.  o_done is at
          // most one phase behind: P_{j-1} was only written after
          // P_{j-2}.V_{j-2} completed.
          if (c == 0 && j > 0) {
            ok = __all_sync(kAll, mbar_wait(o_done, (j - 1) & 1, abort_flag, kWaitLimitNs));
            tc_fence_after();
          }
          // P (16-bit pairs) of score columns 32c..32c+31 -> P columns
          // 16c..16c+15.  Unconditional, so that the exponentials of the next
          // chunk can be scheduled across it; after a failed wait it only
          // writes this CTA's own TMEM columns before the loop is left.
          tmem_st16(pb + 16 * c, pk);
        }
      }
      if (!ok) break;
      bool rescale = false;
      float alpha = 1.f;
      if (__any_sync(kAll, (la[0] + la[1]) + (la[2] + la[3]) > kRowSumBound)) {
        float mm[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) mm[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
        for (int i = 4; i < TN / 2; ++i) mm[i % 4] = fmax3(mm[i % 4], s[2 * i], s[2 * i + 1]);
        const float mx = fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3])) * sl2;
        if (__any_sync(kAll, mx > m)) {
          // Recompute this tile against the new maximum and rescale the
          // state of the earlier tiles (none for the first tile: l is 0 and
          // O is overwritten by the first P.V).  A row sum above the bound
          // implies a P above 2, so this branch always raises m.
          const float mnew = fmaxf(m, mx);
          alpha = ex2(m - mnew);
          l *= alpha;
          m = mnew;
          rescale = j > 0;
          const float nm = -m;
          la[0] = la[1] = la[2] = la[3] = 0.f;
          tmem_wait_st();
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = ex2(fmaf(s[32 * c + 2 * i], sl2, nm));
              const float p1 = ex2(fmaf(s[32 * c + 2 * i + 1], sl2, nm));
              la[i % 4] += p0 + p1;
              pk[i] = pack2<BF16>(p0, p1);
            }
            tmem_st16(pb + 16 * c, pk);
          }
        }
      }
      l += (la[0] + la[1]) + (la[2] + la[3]);
      if (rescale) {
        // O holds the sum over earlier tiles scaled by 2^-m_old.
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
      mbar_arrive(p_full);
    }
    if (ok && n > 0)
      ok = __all_sync(kAll, mbar_wait(o_done, (n - 1) & 1, abort_flag, kWaitLimitNs));
    if (!ok) fail();
    tc_fence_after();
    if (ok && n > 0) {
      const int r = it.qtile * kTileM + row;
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
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool BF16>
cudaError_t launch_t(const AttnParams& p, const void* tq, const void* tkv, const void* tke,
                     const void* tve, cudaStream_t s, Recorder* rec) {
  using C = Cfg<D>;
  auto kern = attn_sm100_kernel<D, BF16>;
  // The shared-memory opt-in is a per-device function attribute: set it once
  // on every device the kernel is launched on.
  constexpr int kMaxDev = 64;
  static bool configured[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  CUtensorMap mq, mkv, mke, mve;
  memcpy(&mq, tq, sizeof(mq));
  memcpy(&mkv, tkv, sizeof(mkv));
  memcpy(&mke, tke ? tke : tq, sizeof(mke));
  memcpy(&mve, tve ? tve : tq, sizeof(mve));
  return dispatch(rec, kern, p.total_items, threads_for(D), C::kSmemBytes, s, mq, mkv, mke, mve,
                  p);
}


}  // namespace

int attn_items_per_stream(int H, int D, int qtiles, int chunks) {
  (void)D;
  return H * qtiles * chunks;
}

int attn_ctas_per_sm(int D) { (void)D; return 2; }   // 256 TMEM columns and < 113 KB smem each

cudaError_t launch_attn_sm100(const AttnParams& p, const void* tmap_q, const void* tmap_kv,
                              const void* tmap_ke, const void* tmap_ve, int dtype,
                              cudaStream_t s, Recorder* rec) {
  if (p.total_items == 0) return cudaSuccess;
  const bool bf16 = dtype == SVT_BF16;
  if (p.D == 64)
    return bf16 ? launch_t<64, true>(p, tmap_q, tmap_kv, tmap_ke, tmap_ve, s, rec)
                : launch_t<64, false>(p, tmap_q, tmap_kv, tmap_ke, tmap_ve, s, rec);
  if (p.D == 128)
    return bf16 ? launch_t<128, true>(p, tmap_q, tmap_kv, tmap_ke, tmap_ve, s, rec)
                : launch_t<128, false>(p, tmap_q, tmap_kv, tmap_ke, tmap_ve, s, rec);
  return cudaErrorInvalidValue;
}

}  // namespace svt
