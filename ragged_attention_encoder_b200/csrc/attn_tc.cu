// Tensor-core attention over 128-row query tiles for sm_100a (tcgen05 + TMEM + TMA).
//
// Serves the paged cross-attention of multi-token query packs (M* page
// "mstar.engine.resources.attn.cross", FlashInferCrossManager.run: non-causal over the
// context) and the cacheless ragged attentions (page "mstar.engine.resources.attn.ragged.base":
// block-causal self-attention within a span, and two-span cross-attention).
//
// A tile is up to 128 query rows of one (request, KV head): rows are (token, head in group)
// pairs, so the g = Hq/Hkv query heads that share a KV head share every K/V byte loaded.
// Per 128-key block j of the tile's key range:
//     S   = Q K^T                     tcgen05.mma, M=128 N=128, fp32 accumulators in TMEM
//     P   = exp2(S*scale*log2e - m)   one thread per row (TMEM lane), fp32, online max
//     O  += P V                       tcgen05.mma, M=128 N=d, P staged as bf16 in smem
// and the epilogue writes O / l as bf16 (or an fp32 partial and its log2-sum-exp when the
// plan split the unit's keys).  The row sum l is accumulated from the bf16-rounded P that
// the tensor core multiplies, so a constant V comes back exactly.
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue (warp w owns TMEM lanes 32w..32w+31),
// warp 4 TMA producer, warp 5 MMA issuer (one thread) and TMEM owner.  K/V blocks stream
// through a 2-stage ring; S of block j+1 is computed while the softmax of block j runs.
// Masking is by select (never by adding): keys past the row's limit get -inf, and V rows past
// the valid keys of the last block are zeroed in shared memory before P.V, so junk (even NaN)
// in page tails cannot reach the output.
#include "kernels.h"
#include "ptx.cuh"

namespace rae {
namespace {

constexpr int kTcThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSCol = 0;
constexpr uint32_t kOCol = 128;
constexpr int kChunkBytes = 128 * 128;   // 128 rows x 64 bf16 (one 128-byte swizzle span)

template <int D>
struct TcLayout {
  static constexpr int CH = D / 64;
  static constexpr int TILE = CH * kChunkBytes;   // Q, K or V tile bytes
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE;
  static constexpr int V_OFF = K_OFF + kStages * TILE;
  static constexpr int P_OFF = V_OFF + kStages * TILE;
  static constexpr int BAR_OFF = P_OFF + 2 * kChunkBytes;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;   // barriers + alignment slack
};

struct TcBars {
  uint64_t q_full, q_empty, s_full, s_free, p_full, pv_done, o_free, fin;
  uint64_t k_full[kStages], v_full[kStages], kv_empty[kStages];
  uint32_t tmem_base;
  int abort;
};

struct TcParams {
  TcTensors maps;
  DevPlan plan;
  Geometry geo;
  __nv_bfloat16* out;
  float* part_o;
  float* part_lse;
  int* err;
  float scale_log2;
  int32_t paged;
  int64_t timeout_ns;
};

__device__ __forceinline__ int tile_blocks(const Tile& t) {
  return (t.kv1 - t.kv0 + kTcBlockKeys - 1) / kTcBlockKeys;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using L = TcLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcBars& bar = *reinterpret_cast<TcBars*>(smem + L::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const DevPlan& plan = p.plan;
  const Geometry& geo = p.geo;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_free, 4);
    mbar_init(&bar.p_full, 4);
    mbar_init(&bar.pv_done, 1);
    mbar_init(&bar.o_free, 4);
    mbar_init(&bar.fin, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
    }
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
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
  const uint32_t tmem = bar.tmem_base;
  const WaitCtl wc{&bar.abort, p.err, p.timeout_ns};

  const int t_begin = plan.cta_ptr[blockIdx.x];
  const int t_end = plan.cta_ptr[blockIdx.x + 1];
  const int g = geo.g;
  const int tpt = kTcRows / g;   // query tokens per tile

  if (warp == 4) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();
      const uint32_t q_bytes = uint32_t(L::CH) * 64u * 2u * uint32_t(g * tpt);
      uint32_t q_use = 0, kv_use = 0;
      for (int t = t_begin; t < t_end && !bar.abort; ++t) {
        const Tile tile = plan.tiles[t];
        const int n = tile_blocks(tile);
        if (n == 0) continue;
        if (q_use > 0 && !wait_bounded(&bar.q_empty, (q_use - 1) & 1, wc, 201)) break;
        mbar_arrive_expect_tx(&bar.q_full, q_bytes);
        for (int c = 0; c < L::CH; ++c)
          tma_load_3d(smem + L::Q_OFF + c * kChunkBytes, &p.maps.q, &bar.q_full, c * 64,
                      tile.kv_head * g, tile.q0, pol_q);
        ++q_use;
        const int32_t* pages = p.paged ? plan.d + plan.c[tile.req] : nullptr;
        const int32_t kv_base = p.paged ? 0 : plan.b[tile.req];
        bool ok = true;
        for (int j = 0; j < n; ++j, ++kv_use) {
          const int s = kv_use % kStages;
          if (kv_use >= uint32_t(kStages) &&
              !wait_bounded(&bar.kv_empty[s], ((kv_use / kStages) - 1) & 1, wc, 202)) {
            ok = false;
            break;
          }
          const int key0 = tile.kv0 + j * kTcBlockKeys;
          uint8_t* ks = smem + L::K_OFF + s * L::TILE;
          uint8_t* vs = smem + L::V_OFF + s * L::TILE;
          if (p.paged) {
            const int P = geo.page_size;
            const int nk = min(kTcBlockKeys, tile.kv1 - key0);
            const int npg = (nk + P - 1) / P;
            const uint32_t bytes = uint32_t(npg) * uint32_t(P) * 128u * L::CH;
            mbar_arrive_expect_tx(&bar.k_full[s], bytes);
            mbar_arrive_expect_tx(&bar.v_full[s], bytes);
            for (int i = 0; i < npg; ++i) {
              const int page = pages[key0 / P + i];
              const int row = (page * geo.hkv + tile.kv_head) * P;
              for (int c = 0; c < L::CH; ++c) {
                tma_load_2d(ks + c * kChunkBytes + i * P * 128, &p.maps.k, &bar.k_full[s], c * 64, row, pol_kv);
                tma_load_2d(vs + c * kChunkBytes + i * P * 128, &p.maps.v, &bar.v_full[s], c * 64, row, pol_kv);
              }
            }
          } else {
            const uint32_t bytes = uint32_t(L::TILE);
            mbar_arrive_expect_tx(&bar.k_full[s], bytes);
            mbar_arrive_expect_tx(&bar.v_full[s], bytes);
            for (int c = 0; c < L::CH; ++c) {
              tma_load_3d(ks + c * kChunkBytes, &p.maps.k, &bar.k_full[s], c * 64, tile.kv_head,
                          kv_base + key0, pol_kv);
              tma_load_3d(vs + c * kChunkBytes, &p.maps.v, &bar.v_full[s], c * 64, tile.kv_head,
                          kv_base + key0, pol_kv);
            }
          }
        }
        if (!ok) break;
      }
      // Drain: every armed copy lands before the CTA may exit.
      const int64_t lim = p.timeout_ns;
      for (uint32_t u = kv_use > uint32_t(kStages) ? kv_use - kStages : 0; u < kv_use; ++u) {
        const int s = u % kStages;
        const uint64_t t0 = global_timer_ns();
        while (!(mbar_try_wait(&bar.k_full[s], (u / kStages) & 1) &&
                 mbar_try_wait(&bar.v_full[s], (u / kStages) & 1)) &&
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
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = sbase + L::Q_OFF;
      const uint32_t p_addr = sbase + L::P_OFF;
      uint32_t q_use = 0, kv_use = 0, blk = 0, o_waits = 0, tiles_done = 0;
      // The P.V of block b is issued after the QK^T of block b+1, so that the tensor core
      // computes the next scores while the softmax of block b runs.
      bool have_prev = false, prev_first = false, prev_wait_o = false;
      uint32_t prev_blk = 0, prev_use = 0;
      auto issue_pv = [&]() -> bool {
        if (!wait_bounded(&bar.p_full, prev_blk & 1, wc, 211)) return false;
        const int s = prev_use % kStages;
        if (!wait_bounded(&bar.v_full[s], (prev_use / kStages) & 1, wc, 212)) return false;
        if (prev_wait_o) {
          if (!wait_bounded(&bar.o_free, o_waits & 1, wc, 213)) return false;
          ++o_waits;
        }
        tc_fence_after();
        const uint32_t v_addr = sbase + L::V_OFF + s * L::TILE;
#pragma unroll
        for (int ks = 0; ks < kTcBlockKeys / 16; ++ks) {
          const uint64_t a = smem_desc_sw128(p_addr + (ks >> 2) * kChunkBytes + (ks & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(v_addr + ks * 16 * 128, kChunkBytes, 1024);
          umma_ss(tmem + kOCol, a, b, idesc_pv, (ks > 0 || !prev_first) ? 1u : 0u);
        }
        umma_commit(&bar.kv_empty[s]);
        umma_commit(&bar.pv_done);
        return true;
      };
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Tile tile = plan.tiles[t];
        const int n = tile_blocks(tile);
        if (n == 0) continue;
        if (!wait_bounded(&bar.q_full, q_use & 1, wc, 214)) { ok = false; break; }
        ++q_use;
        for (int j = 0; j < n; ++j, ++kv_use, ++blk) {
          const int s = kv_use % kStages;
          if (!wait_bounded(&bar.k_full[s], (kv_use / kStages) & 1, wc, 215)) { ok = false; break; }
          if (blk > 0 && !wait_bounded(&bar.s_free, (blk - 1) & 1, wc, 216)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = sbase + L::K_OFF + s * L::TILE;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks >> 2) * kChunkBytes + (ks & 3) * 32;
            const uint64_t a = smem_desc_sw128(q_addr + off, 16, 1024);
            const uint64_t b = smem_desc_sw128(k_addr + off, 16, 1024);
            umma_ss(tmem + kSCol, a, b, idesc_qk, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bar.s_full);
          if (j == n - 1) umma_commit(&bar.q_empty);
          if (have_prev && !issue_pv()) { ok = false; break; }
          have_prev = true;
          prev_blk = blk;
          prev_use = kv_use;
          prev_first = (j == 0);
          prev_wait_o = (j == 0 && tiles_done > 0);
        }
        ++tiles_done;
      }
      if (ok && have_prev) issue_pv();
      // Every issued MMA completes before TMEM is released.
      umma_commit(&bar.fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.fin, 0) && int64_t(global_timer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else {
    // ================================================================ softmax + epilogue
    const int r = warp * 32 + lane;               // tile row == TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(warp * 32) << 16);
    const int tok = r / g;
    const int jh = r - tok * g;
    uint32_t kv_use = 0, blk = 0;
    for (int t = t_begin; t < t_end; ++t) {
      const Tile tile = plan.tiles[t];
      const int n = tile_blocks(tile);
      const bool row_ok = tok < tile.qn && r < tpt * g;
      const int q_tok = tile.q0 + tok;
      const int head = tile.kv_head * g + jh;
      // Keys visible to this row, as a limit on the logical key index.
      int lim = tile.kv1;
      if (!p.paged) {
        const int lk = plan.b[tile.req + 1] - plan.b[tile.req];
        int rl = lk;
        if (plan.block_size > 0) {
          const int i_local = q_tok - plan.a[tile.req];
          const long long end = (long long)(i_local / plan.block_size + 1) * plan.block_size;
          rl = int(min((long long)lk, end));
        }
        lim = min(lim, rl);
      }
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < n; ++j, ++kv_use, ++blk) {
        const int s = kv_use % kStages;
        ok = __all_sync(0xffffffffu, wait_bounded(&bar.s_full, blk & 1, wc, 221));
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + kSCol + c * 32, sv[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_ld(sv[c]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.s_free);

        const int key0 = tile.kv0 + j * kTcBlockKeys;
        const int nv = max(0, min(kTcBlockKeys, lim - key0));
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = c * 32 + e;
            const float x = col < nv ? __uint_as_float(sv[c][e]) * p.scale_log2 : -INFINITY;
            sv[c][e] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        const float mn = fmaxf(m, mx);
        // Rescale lazily: keep the old maximum unless the new one exceeds it by 2^8.
        const bool need = (j == 0) ? true : (mn > m + 8.f);
        const bool warp_need = __any_sync(0xffffffffu, need && j > 0);
        float m_use = need ? mn : m;
        const float corr = (need && m != -INFINITY && mn != -INFINITY) ? fast_exp2(m - mn)
                                                                      : (need && j > 0 ? 0.f : 1.f);
        const float base = (m_use == -INFINITY) ? 0.f : m_use;
        float psum = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = fast_exp2(__uint_as_float(sv[c][e]) - base);
            const float p1 = fast_exp2(__uint_as_float(sv[c][e + 1]) - base);
            const uint32_t w = pack_bf16x2(p0, p1);
            pk[c * 16 + e / 2] = w;
            psum += bf16lo_to_f32(w) + bf16hi_to_f32(w);
          }
        if (blk > 0) {
          ok = __all_sync(0xffffffffu, wait_bounded(&bar.pv_done, (blk - 1) & 1, wc, 222));
          if (!ok) break;
        }
        if (warp_need) {
          tc_fence_after();
          const float cf = (need && j > 0) ? corr : 1.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(lane_addr + kOCol + c * 32, ov);
            tmem_wait_ld(ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * cf);
            tmem_st32(lane_addr + kOCol + c * 32, ov);
          }
          tmem_wait_st();
        }
        l = (j > 0 && need) ? l * corr + psum : (j == 0 ? psum : l + psum);
        m = m_use;
        // P row r -> bf16, 128-byte swizzled K-major layout (two 64-key chunks).
        uint8_t* prow = smem + L::P_OFF + r * 128;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int chunk = u >> 3, w = u & 7;
          uint4 v;
          v.x = pk[u * 4 + 0];
          v.y = pk[u * 4 + 1];
          v.z = pk[u * 4 + 2];
          v.w = pk[u * 4 + 3];
          *reinterpret_cast<uint4*>(prow + chunk * kChunkBytes + ((w ^ (r & 7)) << 4)) = v;
        }
        // V rows past the block's valid keys hold stale or junk data: zero them.
        const int vb = min(kTcBlockKeys, tile.kv1 - key0);
        if (r >= vb) {
          if (wait_bounded(&bar.v_full[s], (kv_use / kStages) & 1, wc, 223)) {
            uint8_t* vrow = smem + L::V_OFF + s * L::TILE + r * 128;
#pragma unroll
            for (int c = 0; c < L::CH; ++c)
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(vrow + c * kChunkBytes + u * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      const bool split = tile.part >= 0;
      if (n > 0) {
        ok = __all_sync(0xffffffffu, wait_bounded(&bar.pv_done, (blk - 1) & 1, wc, 224));
        if (!ok) break;
        tc_fence_after();
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (n > 0) {
          tmem_ld32(lane_addr + kOCol + c * 32, ov);
          tmem_wait_ld(ov);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0u;
        }
        if (!row_ok) continue;
        if (!split) {
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pkd[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t(q_tok) * geo.hq + head) * D + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
        } else {
          float4* dst = reinterpret_cast<float4*>(p.part_o + int64_t(tile.part + r) * D + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                 __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
        }
      }
      if (split && row_ok) p.part_lse[tile.part + r] = l > 0.f ? m + fast_log2(l) : -INFINITY;
      if (n > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.o_free);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_tc(const DevPlan& plan, const Geometry& geo, bool paged,
                           const TcTensors& maps, void* out, float* part_o, float* part_lse,
                           int* err, float scale_log2, int64_t timeout_ns, cudaStream_t stream) {
  if (plan.num_ctas == 0) return cudaSuccess;
  TcParams prm;
  prm.maps = maps;
  prm.plan = plan;
  prm.geo = geo;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.part_o = part_o;
  prm.part_lse = part_lse;
  prm.err = err;
  prm.scale_log2 = scale_log2;
  prm.paged = paged ? 1 : 0;
  prm.timeout_ns = timeout_ns;
  cudaError_t e;
  if (geo.d == 128) {
    e = cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TcLayout<128>::SMEM);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<128><<<dim3(uint32_t(plan.num_ctas)), kTcThreads, TcLayout<128>::SMEM, stream>>>(prm);
  } else {
    e = cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TcLayout<64>::SMEM);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<64><<<dim3(uint32_t(plan.num_ctas)), kTcThreads, TcLayout<64>::SMEM, stream>>>(prm);
  }
  return cudaGetLastError();
}

}  // namespace rae
