// Paged cross-attention for a few query rows per (request, KV head) on tcgen05, with the
// operands swapped so that the 128 keys of a block fill the MMA's M dimension.
//
// M* page "mstar.engine.resources.attn.cross" (FlashInferCrossManager.run): non-causal
// attention of packed decoder queries over the context pages.  With 9..64 query rows per
// (request, KV head) -- e.g. 4 tokens x 8 GQA heads -- a 128-row query tile would be mostly
// padding and every softmax thread would exponentiate 128 keys.  Here, per 128-key block j:
//     S^T = K_j Q^T          tcgen05.mma M=128 (keys) N=rows, fp32 in TMEM (double-buffered)
//     P^T = 2^(S^T*scale*log2e - m)   one thread per key: N exponentials, not 128
//     O^T += V_j^T P^T       tcgen05.mma M=128 (= d) N=rows, V^T read MN-major from the same
//                            shared-memory tile, P^T staged bf16 in 64-byte-swizzled smem
// Column (= query row) maxima and sums need all 128 keys: a warp transpose-reduction (31
// shuffles for 32 columns) and an exchange of the four warps' results through shared memory.
// O is rescaled only when a column's maximum grows by more than 2^8.  The tile writes O^T / l
// transposed (consecutive lanes hold consecutive head dimensions, so stores stay coalesced),
// or fp32 partials plus log2-sum-exp when the plan split the unit's keys; the CTA completing
// a unit's last split merges it (merge.cuh).
//
// Warp roles (192 threads): warps 0-3 softmax / epilogue (warp w owns TMEM lanes 32w..+31:
// keys for S^T, head dimensions for O^T), warp 4 TMA producer, warp 5 MMA issuer and TMEM
// owner.  Three K/V stages keep 192 KB of loads in flight per SM; the path is HBM bound.
#include "kernels.h"
#include "merge.cuh"
#include "ptx.cuh"

namespace rae {
namespace {

constexpr int kSwThreads = 192;
constexpr int kD = 128;                 // head dimension of this kernel
constexpr int kKvTile = 128 * kD * 2;   // bytes of a 128-key K or V tile (two 64-wide chunks)
constexpr int kChunk = 128 * 128;

template <int N>
struct SwLayout {
  static_assert(N == 32 || N == 64, "query rows per tile");
  static constexpr int STAGES = N == 32 ? 3 : 2;
  static constexpr int QCH = N * 128;                 // one 64-wide chunk of Q (N rows)
  static constexpr int PROW = N * 2;                  // bytes of a key's row of P^T
  static constexpr int PBUF = 128 * PROW;             // one P^T buffer
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = 2 * QCH < 1024 ? 1024 : 2 * QCH;
  static constexpr int V_OFF = K_OFF + STAGES * kKvTile;
  static constexpr int P_OFF = V_OFF + STAGES * kKvTile;
  static constexpr int BAR_OFF = P_OFF + 2 * PBUF;
  static constexpr int SMEM = BAR_OFF + 2048 + 1024;  // barriers, reduction scratch, slack
  static constexpr uint32_t TMEM_COLS = 4 * N <= 128 ? 128 : 256;   // S^T x2, O^T
  static constexpr uint32_t O_COL = 2 * N;
  // MN-major swizzle of P^T: 64-byte rows (SW64) for 32 rows, 128-byte rows (SW128) for 64.
  static constexpr uint32_t P_SWIZZLE = N == 32 ? 4u : 2u;
  static constexpr uint32_t P_SBO = N == 32 ? 512u : 1024u;
};

struct SwBars {
  uint64_t q_full, q_empty, fin, merge_in, merge_out;
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], o_free;
  uint64_t k_full[3], v_full[3], kv_empty[3];
  uint32_t tmem_base;
  int merge_flag;
  int abort;
  int any_rescale;
};

struct SwParams {
  TcTensors maps;
  DevPlan plan;
  Geometry geo;
  __nv_bfloat16* out;
  float* part_o;
  float* part_lse;
  int* err;
  float scale_log2;
  int64_t timeout_ns;
};

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t((lbo >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(layout) << 61;
  return d;
}

// Column-wise reduction of a warp: on entry every lane holds 32 values v[c] (one per column);
// on exit lane l holds the reduction of column l over the warp's 32 lanes.
template <bool IS_MAX>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const bool upper = lane & w;
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

template <int N>
__global__ void __launch_bounds__(kSwThreads, 1) attn_swapab_kernel(const __grid_constant__ SwParams p) {
  using L = SwLayout<N>;
  constexpr int NG = N / 32;   // groups of 32 columns
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SwBars& bar = *reinterpret_cast<SwBars*>(smem + L::BAR_OFF);
  float* red = reinterpret_cast<float*>(smem + L::BAR_OFF + 512);   // [4][N] per-warp results
  float* mcur = red + 4 * N;                                        // [N] exponent base
  float* corr = mcur + N;                                           // [N] rescale factor
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const DevPlan& plan = p.plan;
  const Geometry& geo = p.geo;
  const int g = geo.g;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.merge_in, 4);
    mbar_init(&bar.merge_out, 1);
    mbar_init(&bar.o_free, 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.s_full[b], 1);
      mbar_init(&bar.s_free[b], 4);
      mbar_init(&bar.p_full[b], 4);
      mbar_init(&bar.pv_done[b], 1);
    }
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
    }
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar.tmem_base, L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&p.maps.q);
    prefetch_tmap(&p.maps.k);
    prefetch_tmap(&p.maps.v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t tmem = bar.tmem_base;
  const WaitCtl wc{&bar.abort, p.err, p.timeout_ns};
  const int t_begin = plan.cta_ptr[blockIdx.x];
  const int t_end = plan.cta_ptr[blockIdx.x + 1];

  if (warp == 4) {
    // ================================================================ TMA producer
    // The whole warp walks the tiles: lane 0 takes the barrier waits and arms the transaction
    // counts; lane i reads the page id of the block's i-th page (before the stage's empty
    // wait, so those reads overlap it) and issues that page's copies.
    const uint64_t pol_q = policy_evict_first();
    const uint64_t pol_kv = policy_evict_first();
    uint32_t q_use = 0, kv_use = 0;
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Tile tile = plan.tiles[t];
      const int n = (tile.kv1 - tile.kv0 + kTcBlockKeys - 1) / kTcBlockKeys;
      if (n == 0) continue;
      if (lane == 0) {
        if (q_use > 0 && !wait_bounded(&bar.q_empty, (q_use - 1) & 1, wc, 401)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(&bar.q_full, 2u * L::QCH);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(smem + L::Q_OFF + c * L::QCH, &p.maps.q, &bar.q_full, c * 64,
                        tile.kv_head * g, tile.q0, pol_q);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++q_use;
      const int32_t* pages = plan.d + plan.c[tile.req];
      const int P = geo.page_size;
      for (int j = 0; j < n; ++j, ++kv_use) {
        const int s = kv_use % L::STAGES;
        const int key0 = tile.kv0 + j * kTcBlockKeys;
        const int npg = (min(kTcBlockKeys, tile.kv1 - key0) + P - 1) / P;   // <= 8 pages
        const uint32_t bytes = uint32_t(npg) * uint32_t(P) * 256u;
        const int row = lane < npg ? (pages[key0 / P + lane] * geo.hkv + tile.kv_head) * P : 0;
        if (lane == 0) {
          if (kv_use >= uint32_t(L::STAGES) &&
              !wait_bounded(&bar.kv_empty[s], ((kv_use / L::STAGES) - 1) & 1, wc, 402)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(&bar.k_full[s], bytes);
            mbar_arrive_expect_tx(&bar.v_full[s], bytes);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane < npg) {
          uint8_t* ks = smem + L::K_OFF + s * kKvTile + lane * P * 128;
          uint8_t* vs = smem + L::V_OFF + s * kKvTile + lane * P * 128;
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(ks + c * kChunk, &p.maps.k, &bar.k_full[s], c * 64, row, pol_kv);
            tma_load_2d(vs + c * kChunk, &p.maps.v, &bar.v_full[s], c * 64, row, pol_kv);
          }
        }
      }
    }
    if (lane == 0) {
      const int64_t lim = p.timeout_ns;
      for (uint32_t u = kv_use > uint32_t(L::STAGES) ? kv_use - L::STAGES : 0; u < kv_use; ++u) {
        const int s = u % L::STAGES;
        const uint64_t t0 = global_timer_ns();
        while (!(mbar_try_wait(&bar.k_full[s], (u / L::STAGES) & 1) &&
                 mbar_try_wait(&bar.v_full[s], (u / L::STAGES) & 1)) &&
               int64_t(global_timer_ns() - t0) < lim) {
        }
      }
      if (q_use > 0) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.q_full, (q_use - 1) & 1) && int64_t(global_timer_ns() - t0) < lim) {
        }
      }
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      // S^T: A = K (keys x d, K-major), B = Q (rows x d, K-major).
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, N, false, false);
      // O^T: A = V^T (d x keys, MN-major), B = P^T (keys x rows, MN-major).
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, N, true, true);
      uint32_t q_use = 0, kv_use = 0, s_use[2] = {0, 0}, p_use[2] = {0, 0}, tiles_done = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t use, int b) -> bool {
        const int s = use % L::STAGES;
        if (!wait_bounded(&bar.k_full[s], (use / L::STAGES) & 1, wc, 411)) return false;
        if (s_use[b] > 0 && !wait_bounded(&bar.s_free[b], (s_use[b] - 1) & 1, wc, 412)) return false;
        tc_fence_after();
        const uint32_t k_addr = sbase + L::K_OFF + s * kKvTile;
        const uint32_t q_addr = sbase + L::Q_OFF;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t a = smem_desc(k_addr + (ks >> 2) * kChunk + (ks & 3) * 32, 16, 1024, 2);
          const uint64_t bq = smem_desc(q_addr + (ks >> 2) * L::QCH + (ks & 3) * 32, 16, 1024, 2);
          umma_ss(tmem + uint32_t(b) * N, a, bq, idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bar.s_full[b]);
        ++s_use[b];
        return true;
      };
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Tile tile = plan.tiles[t];
        const int n = (tile.kv1 - tile.kv0 + kTcBlockKeys - 1) / kTcBlockKeys;
        if (n == 0) continue;
        if (!wait_bounded(&bar.q_full, q_use & 1, wc, 413)) { ok = false; break; }
        ++q_use;
        if (!issue_s(kv_use, 0)) { ok = false; break; }
        if (n == 1) umma_commit(&bar.q_empty);
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t use = kv_use + j;
          const int b = j & 1;
          if (j + 1 < n) {
            if (!issue_s(use + 1, (j + 1) & 1)) { ok = false; break; }
            if (j + 2 == n) umma_commit(&bar.q_empty);
          }
          const int s = use % L::STAGES;
          if (!wait_bounded(&bar.p_full[b], p_use[b] & 1, wc, 414)) { ok = false; break; }
          if (!wait_bounded(&bar.v_full[s], (use / L::STAGES) & 1, wc, 415)) { ok = false; break; }
          if (j == 0 && tiles_done > 0 && !wait_bounded(&bar.o_free, (tiles_done - 1) & 1, wc, 416)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_addr = sbase + L::V_OFF + s * kKvTile;
          const uint32_t p_addr = sbase + L::P_OFF + b * L::PBUF;
#pragma unroll
          for (int ks = 0; ks < kTcBlockKeys / 16; ++ks) {
            const uint64_t a = smem_desc(v_addr + ks * 16 * 128, kChunk, 1024, 2);
            const uint64_t bp = smem_desc(p_addr + ks * 16 * L::PROW, 16, L::P_SBO, L::P_SWIZZLE);
            umma_ss(tmem + L::O_COL, a, bp, idesc_o, (ks > 0 || j > 0) ? 1u : 0u);
          }
          umma_commit(&bar.kv_empty[s]);
          umma_commit(&bar.pv_done[b]);
          ++p_use[b];
        }
        kv_use += n;
        ++tiles_done;
      }
      umma_commit(&bar.fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.fin, 0) && int64_t(global_timer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else {
    // ================================================================ softmax + epilogue
    const int k = warp * 32 + lane;   // key of S^T / head dimension of O^T (TMEM lane)
    const uint32_t lane_addr = tmem + (uint32_t(warp * 32) << 16);
    uint32_t kv_use = 0, s_use[2] = {0, 0}, p_use[2] = {0, 0}, split_seen = 0, tiles_done = 0;
    bool ok = true;
    for (int t = t_begin; t < t_end; ++t) {
      const Tile tile = plan.tiles[t];
      const int n = (tile.kv1 - tile.kv0 + kTcBlockKeys - 1) / kTcBlockKeys;
      const int rows = tile.qn * g;
      float lsum[N];
#pragma unroll
      for (int c = 0; c < N; ++c) lsum[c] = 0.f;
      float m_own = -INFINITY;   // exponent base of column k (threads k < N)
      for (int j = 0; j < n; ++j) {
        const uint32_t use = kv_use + j;
        const int b = j & 1;
        // A failed wait only disables work: every warp keeps executing the same sequence of
        // named barriers, so no warp can be left waiting at one.
        ok = __all_sync(0xffffffffu, ok && wait_bounded(&bar.s_full[b], s_use[b] & 1, wc, 421));
        ++s_use[b];
        tc_fence_after();
        float x[N];
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          uint32_t r32[32];
          if (ok) {
            tmem_ld32(lane_addr + uint32_t(b) * N + gq * 32, r32);
            tmem_wait_ld(r32);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) r32[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) x[gq * 32 + c] = __uint_as_float(r32[c]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.s_free[b]);
        const int key0 = tile.kv0 + j * kTcBlockKeys;
        const bool valid = key0 + k < tile.kv1;
#pragma unroll
        for (int c = 0; c < N; ++c) x[c] = valid ? x[c] * p.scale_log2 : -INFINITY;
        // Column maxima over the 128 keys.
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          float v[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = x[gq * 32 + c];
          red[warp * N + gq * 32 + lane] = warp_transpose_reduce<true>(v, lane);
        }
        named_bar_sync(1, 128);
        if (k < N) {
          const float mx = fmaxf(fmaxf(red[k], red[N + k]), fmaxf(red[2 * N + k], red[3 * N + k]));
          const float mn = fmaxf(m_own, mx);
          // Keep the old base unless the new maximum exceeds it by 2^8 (exact after division).
          const bool need = (j == 0) || (mn > m_own + 8.f);
          const float cf = (j > 0 && need && m_own != -INFINITY) ? fast_exp2(m_own - mn) : 1.f;
          if (need) m_own = mn;
          mcur[k] = m_own == -INFINITY ? 0.f : m_own;
          corr[k] = cf;
        }
        if (k == 0) bar.any_rescale = 0;
        named_bar_sync(1, 128);
        if (k < N && corr[k] != 1.f) bar.any_rescale = 1;
        // p = 2^(x - m) for this key across the columns; per-key partial row sums.
        float pv[N];
#pragma unroll
        for (int c = 0; c < N; ++c) {
          pv[c] = fast_exp2(x[c] - mcur[c]);
          lsum[c] = lsum[c] * corr[c] + pv[c];
        }
        named_bar_sync(1, 128);
        const bool rescale = bar.any_rescale != 0;
        // P^T buffer b is free once P.V two blocks back has completed.
        if (p_use[b] > 0)
          ok = __all_sync(0xffffffffu, ok && wait_bounded(&bar.pv_done[b], (p_use[b] - 1) & 1, wc, 422));
        if (rescale && j > 0) {
          // O^T holds the sum through block j-1 once its P.V has completed.
          const int pb = (j - 1) & 1;
          ok = __all_sync(0xffffffffu, ok && wait_bounded(&bar.pv_done[pb], (p_use[pb] - 1) & 1, wc, 423));
        }
        if (ok && rescale && j > 0) {
          tc_fence_after();
#pragma unroll
          for (int gq = 0; gq < NG; ++gq) {
            uint32_t ov[32];
            tmem_ld32(lane_addr + L::O_COL + gq * 32, ov);
            tmem_wait_ld(ov);
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * corr[gq * 32 + c]);
            tmem_st32(lane_addr + L::O_COL + gq * 32, ov);
          }
          tmem_wait_st();
        }
        // P^T row k (N bf16) into the swizzled MN-major buffer.
        uint8_t* prow = smem + L::P_OFF + b * L::PBUF + k * L::PROW;
#pragma unroll
        for (int u = 0; u < L::PROW / 16; ++u) {
          uint4 w;
          w.x = pack_bf16x2(pv[8 * u + 0], pv[8 * u + 1]);
          w.y = pack_bf16x2(pv[8 * u + 2], pv[8 * u + 3]);
          w.z = pack_bf16x2(pv[8 * u + 4], pv[8 * u + 5]);
          w.w = pack_bf16x2(pv[8 * u + 6], pv[8 * u + 7]);
          const int pu = N == 32 ? (u ^ ((k >> 1) & 3)) : (u ^ (k & 7));
          *reinterpret_cast<uint4*>(prow + pu * 16) = w;
        }
        // V rows past the block's valid keys hold stale or junk data: zero them.
        if (!valid) {
          const int s = use % L::STAGES;
          if (wait_bounded(&bar.v_full[s], (use / L::STAGES) & 1, wc, 424)) {
            uint8_t* vrow = smem + L::V_OFF + s * kKvTile + k * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(vrow + c * kChunk + u * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full[b]);
        ++p_use[b];
      }
      kv_use += n;
      // ---------------------------------------------------------------- epilogue
      // Row sums: per-key partials reduced over the 128 keys.
#pragma unroll
      for (int gq = 0; gq < NG; ++gq) {
        float v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = lsum[gq * 32 + c];
        red[warp * N + gq * 32 + lane] = warp_transpose_reduce<false>(v, lane);
      }
      named_bar_sync(1, 128);
      if (k < N) {
        const float l = (red[k] + red[N + k]) + (red[2 * N + k] + red[3 * N + k]);
        corr[k] = l > 0.f ? 1.f / l : 0.f;                   // 1 / l per column
        if (tile.part >= 0 && k < rows)
          p.part_lse[tile.part + k] = l > 0.f ? m_own + fast_log2(l) : -INFINITY;
      }
      named_bar_sync(1, 128);
      if (n > 0) {
        const int lb = (n - 1) & 1;
        ok = __all_sync(0xffffffffu, ok && wait_bounded(&bar.pv_done[lb], (p_use[lb] - 1) & 1, wc, 425));
        tc_fence_after();
      }
#pragma unroll
      for (int gq = 0; gq < NG; ++gq) {
        uint32_t ov[32];
        if (n > 0 && ok) {
          tmem_ld32(lane_addr + L::O_COL + gq * 32, ov);
          tmem_wait_ld(ov);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = gq * 32 + c;
          if (col >= rows || !ok) continue;
          const float o = __uint_as_float(ov[c]) * corr[col];
          if (tile.part < 0) {
            const int tok = tile.q0 + col / g;
            const int head = tile.kv_head * g + col % g;
            p.out[(int64_t(tok) * geo.hq + head) * kD + k] = __float2bfloat16_rn(o);
          } else {
            p.part_o[int64_t(tile.part + col) * kD + k] = o;
          }
        }
      }
      if (n > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.o_free);
        ++tiles_done;
      }
      named_bar_sync(1, 128);   // corr[] is reused by the next tile
      if (tile.part >= 0 &&
          split_unit_complete(plan.counters, tile, &bar.merge_in, &bar.merge_out, &bar.merge_flag,
                              split_seen++, threadIdx.x == 0, lane, wc, &ok) && ok)
        merge_split_unit<kD, 4>(tile, geo, tile.kv_head * geo.g, geo.g, p.part_o, p.part_lse, p.out,
                                threadIdx.x, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int N>
cudaError_t launch_n(const SwParams& prm, int num_ctas, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(attn_swapab_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SwLayout<N>::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_swapab_kernel<N>, dim3(uint32_t(num_ctas)), dim3(kSwThreads),
                    SwLayout<N>::SMEM, stream, prm);
}

}  // namespace

cudaError_t launch_attn_swapab(const DevPlan& plan, const Geometry& geo, int n_rows,
                               const TcTensors& maps, void* out, float* part_o, float* part_lse,
                               int* err, float scale_log2, int64_t timeout_ns, cudaStream_t stream) {
  if (plan.num_ctas == 0) return cudaSuccess;
  SwParams prm;
  prm.maps = maps;
  prm.plan = plan;
  prm.geo = geo;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.part_o = part_o;
  prm.part_lse = part_lse;
  prm.err = err;
  prm.scale_log2 = scale_log2;
  prm.timeout_ns = timeout_ns;
  return n_rows == 32 ? launch_n<32>(prm, plan.num_ctas, stream)
                      : launch_n<64>(prm, plan.num_ctas, stream);
}

}  // namespace rae
