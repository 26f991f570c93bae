// Tensor-core attention for sm_100a (tcgen05 + TMEM + TMA), two query tiles per CTA.
//
// Serves the paged cross-attention of multi-token query packs (M* page
// "mstar.engine.resources.attn.cross", FlashInferCrossManager.run: non-causal over the
// context) and the cacheless ragged attentions (page "mstar.engine.resources.attn.ragged.base":
// block-causal self-attention within a span, and two-span cross-attention).
//
// A work tile holds up to two 128-row query tiles Q0, Q1 of one (request, KV head) with one
// key range, so every K/V block loaded serves 256 query rows.  Rows are (token, head in
// group) pairs: the g = Hq/Hkv heads of a KV head share each K/V byte.  Per 128-key block j:
//     S_t = Q_t K_j^T                    tcgen05.mma M=128 N=128, fp32 accumulators in TMEM
//     P_t = exp2(S_t*scale*log2e - m_t)  one thread per row, fp32, written back into TMEM as
//                                        bf16 over the first half of S_t's columns
//     O_t += P_t V_j                     tcgen05.mma with A = P_t read from TMEM, N = d
// The MMA warp interleaves the two tiles (S0 S1 | PV0 S0' | PV1 S1' | ...) so that the tensor
// core works on one tile while the other tile's softmax runs.  O is rescaled only when a row's
// maximum grows by more than 2^8 (the exponent base stays stale otherwise, which is exact
// after the final division).  The row sum l adds the fp32 probabilities; the tensor core
// multiplies their bf16 roundings.
//
// Warp roles (320 threads): warps 0-3 softmax + epilogue of Q0 (TMEM lanes 32w..32w+31),
// warps 4-7 the same for Q1, warp 8 TMA producer, warp 9 MMA issuer and TMEM owner.
// Masking is by select: keys past a row's limit get -inf, and V rows past the valid keys of
// the last block are zeroed in shared memory before P.V, so junk (even NaN) in page tails
// cannot reach the output.  Every wait is bounded.
#include "kernels.h"
#include "merge.cuh"
#include "ptx.cuh"

namespace rae {
namespace {

constexpr int kTcThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStages = 2;
// Q tiles sit in a ring of three slots: the next unit's first Q tile loads while the current
// unit still runs (its slot was released by the unit before), the second as soon as the
// current unit's last S of tile 0 has read that tile's slot.
constexpr int kQSlots = 3;
constexpr uint32_t kTmemCols = 512;
constexpr int kChunkBytes = 128 * 128;   // 128 rows x 64 bf16 (one 128-byte swizzle span)


template <int D>
struct TcLayout {
  static constexpr int CH = D / 64;
  static constexpr int TILE = CH * kChunkBytes;   // bytes of a 128-row Q, K or V tile
  static constexpr int Q_OFF = 0;                  // the ring of Q tile slots
  static constexpr int K_OFF = kQSlots * TILE;
  static constexpr int V_OFF = K_OFF + kStages * TILE;
  static constexpr int BAR_OFF = V_OFF + kStages * TILE;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;   // barriers + alignment slack
  static_assert(SMEM <= 232448, "shared memory of one CTA (227 KB)");
  // TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 after it.
  static __device__ __forceinline__ constexpr uint32_t s_col(int qt) { return uint32_t(qt) * 128u; }
  static __device__ __forceinline__ constexpr uint32_t o_col(int qt) { return 256u + uint32_t(qt) * D; }
};

struct TcBars {
  uint64_t q_full[kQSlots], q_empty[kQSlots], fin;
  uint64_t merge_in, merge_out;   // split-unit arrival protocol (softmax warps)
  int merge_flag;
  uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
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
  int32_t wide_stores;   // out and the partials are 32-byte aligned: one sector per store
  int64_t timeout_ns;
};

__device__ __forceinline__ int tile_blocks(const Tile& t) {
  return (t.kv1 - t.kv0 + kTcBlockKeys - 1) / kTcBlockKeys;
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16 (A = P in TMEM, bf16 pairs per 32-bit column).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// S = Q K^T for one 128-row tile: D/16 MMAs of K=16 over the 128-byte-swizzled K-major tiles.
template <int D>
__device__ __forceinline__ void mma_s(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr,
                                      uint32_t idesc) {
  const uint64_t qd = smem_desc_sw128(q_addr, 16, 1024);
  const uint64_t kd = smem_desc_sw128(k_addr, 16, 1024);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint32_t off = (ks >> 2) * kChunkBytes + (ks & 3) * 32;
    umma_ss(d_tmem, qd + (off >> 4), kd + (off >> 4), idesc, ks > 0 ? 1u : 0u);
  }
}

// O (+)= P V for one tile: P (128 x 128 keys, bf16 pairs) from TMEM, V MN-major from smem.
template <int D>
__device__ __forceinline__ void mma_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_addr,
                                       uint32_t idesc, bool first) {
  const uint64_t vd = smem_desc_sw128(v_addr, kChunkBytes, 1024);
#pragma unroll
  for (int ks = 0; ks < kTcBlockKeys / 16; ++ks)
    umma_ts(o_tmem, p_tmem + ks * 8, vd + uint64_t((ks * 16 * 128) >> 4), idesc,
            (ks > 0 || !first) ? 1u : 0u);
}

// O row *= f, 16 columns at a time (rare: only when a row's maximum grew by more than 2^8).
// Kept out of line so that its registers do not add to the softmax loop's.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t o_addr, float f) {
#pragma unroll 1
  for (int c = 0; c < D / 16; ++c) {
    uint32_t ov[16];
    tmem_ld16(o_addr + c * 16, ov);
    tmem_wait_ld(ov);
#pragma unroll
    for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
    tmem_st16(o_addr + c * 16, ov);
  }
}

// The split merge, kept out of line so that its registers do not add to the softmax loop's.
template <int D>
__device__ __noinline__ void merge_unit(const Tile& tile, const Geometry& geo, const float* part_o,
                                        const float* part_lse, __nv_bfloat16* out) {
  merge_split_unit<D, 8>(tile, geo, tile.kv_head * geo.g, geo.g, part_o, part_lse, out, threadIdx.x, 256);
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
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(&bar.q_full[i], 1);
      mbar_init(&bar.q_empty[i], 1);
    }
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.merge_in, 8);
    mbar_init(&bar.merge_out, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar.s_full[t], 1);
      mbar_init(&bar.p_full[t], 4);
      mbar_init(&bar.pv_done[t], 1);
      mbar_init(&bar.o_free[t], 4);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
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
  const int g = geo.g;
  const int tpt = kTcRows / g;   // query tokens per 128-row tile

  if (warp == kProducerWarp) {
    // ================================================================ TMA producer
    // The whole warp walks the tiles.  Lane 0 takes the barrier waits and arms the
    // transaction counts; for paged K/V, lane i reads the page id of the block's i-th page
    // (before the stage's empty wait, so those reads overlap it and each other) and issues
    // that page's copies.
    const uint64_t pol_q = policy_evict_first();
    const uint64_t pol_kv = policy_evict_last();
    const uint32_t q_tile_bytes = uint32_t(L::CH) * 64u * 2u * uint32_t(g * tpt);
    uint32_t q_cnt = 0, kv_use = 0;   // Q tiles armed; K/V blocks
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Tile tile = plan.tiles[t];
      const int n = tile_blocks(tile);
      if (n == 0) continue;
      const bool has1 = tile.qn > tpt;
      if (lane == 0) {
        for (int qt = 0; qt < (has1 ? 2 : 1); ++qt) {
          const int qs = int(q_cnt % kQSlots);
          if (q_cnt >= uint32_t(kQSlots) &&
              !wait_bounded(&bar.q_empty[qs], ((q_cnt / kQSlots) - 1) & 1, wc, 201)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar.q_full[qs], q_tile_bytes);
          for (int c = 0; c < L::CH; ++c)
            tma_load_3d(smem + L::Q_OFF + qs * L::TILE + c * kChunkBytes, &p.maps.q, &bar.q_full[qs],
                        c * 64, tile.kv_head * g, tile.q0 + qt * tpt, pol_q);
          ++q_cnt;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      q_cnt = __shfl_sync(0xffffffffu, q_cnt, 0);
      if (!ok) break;
      const int32_t* pages = p.paged ? plan.d + plan.c[tile.req] : nullptr;
      const int32_t kv_base = p.paged ? 0 : plan.b[tile.req];
      for (int j = 0; j < n; ++j, ++kv_use) {
        const int s = kv_use % kStages;
        const uint32_t ph = ((kv_use / kStages) - 1) & 1;
        const int key0 = tile.kv0 + j * kTcBlockKeys;
        uint8_t* ks = smem + L::K_OFF + s * L::TILE;
        uint8_t* vs = smem + L::V_OFF + s * L::TILE;
        int npg = 0, row = 0;
        uint32_t bytes = uint32_t(L::TILE);
        if (p.paged) {
          const int P = geo.page_size;
          npg = (min(kTcBlockKeys, tile.kv1 - key0) + P - 1) / P;   // <= 8 pages
          bytes = uint32_t(npg) * uint32_t(P) * 128u * L::CH;
          if (lane < npg) row = (pages[key0 / P + lane] * geo.hkv + tile.kv_head) * P;
        }
        if (lane == 0) {
          if (kv_use >= uint32_t(kStages) && !wait_bounded(&bar.k_empty[s], ph, wc, 202)) ok = false;
          else mbar_arrive_expect_tx(&bar.k_full[s], bytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (p.paged) {
          if (lane < npg)
            for (int c = 0; c < L::CH; ++c)
              tma_load_2d(ks + c * kChunkBytes + lane * geo.page_size * 128, &p.maps.k, &bar.k_full[s],
                          c * 64, row, pol_kv);
        } else if (lane == 0) {
          for (int c = 0; c < L::CH; ++c)
            tma_load_3d(ks + c * kChunkBytes, &p.maps.k, &bar.k_full[s], c * 64, tile.kv_head,
                        kv_base + key0, pol_kv);
        }
        if (lane == 0) {
          if (kv_use >= uint32_t(kStages) && !wait_bounded(&bar.v_empty[s], ph, wc, 203)) {
            ok = false;
            // This stage's K copies are in flight: they land before the CTA may exit.
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&bar.k_full[s], (kv_use / kStages) & 1) &&
                   int64_t(global_timer_ns() - t0) < p.timeout_ns) {
            }
          } else {
            mbar_arrive_expect_tx(&bar.v_full[s], bytes);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (p.paged) {
          if (lane < npg)
            for (int c = 0; c < L::CH; ++c)
              tma_load_2d(vs + c * kChunkBytes + lane * geo.page_size * 128, &p.maps.v, &bar.v_full[s],
                          c * 64, row, pol_kv);
        } else if (lane == 0) {
          for (int c = 0; c < L::CH; ++c)
            tma_load_3d(vs + c * kChunkBytes, &p.maps.v, &bar.v_full[s], c * 64, tile.kv_head,
                        kv_base + key0, pol_kv);
        }
      }
    }
    // Drain: every armed copy lands before the CTA may exit.
    if (lane == 0) {
      const int64_t lim = p.timeout_ns;
      for (uint32_t u = kv_use > uint32_t(kStages) ? kv_use - kStages : 0; u < kv_use; ++u) {
        const int s = u % kStages;
        const uint64_t t0 = global_timer_ns();
        while (!(mbar_try_wait(&bar.k_full[s], (u / kStages) & 1) &&
                 mbar_try_wait(&bar.v_full[s], (u / kStages) & 1)) &&
               int64_t(global_timer_ns() - t0) < lim) {
        }
      }
      for (uint32_t c = q_cnt > uint32_t(kQSlots) ? q_cnt - kQSlots : 0; c < q_cnt; ++c) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.q_full[c % kQSlots], (c / kQSlots) & 1) &&
               int64_t(global_timer_ns() - t0) < lim) {
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      uint32_t q_cnt = 0, kv_use = 0;
      uint32_t pv_cnt0 = 0, pv_cnt1 = 0, o_tiles0 = 0, o_tiles1 = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Tile tile = plan.tiles[t];
        const int n = tile_blocks(tile);
        if (n == 0) continue;
        const bool has1 = tile.qn > tpt;
        // Q slot of each tile of this unit, and its shared-memory address
        const int qs[2] = {int(q_cnt % kQSlots), int((q_cnt + 1) % kQSlots)};
        const uint32_t qa[2] = {sbase + L::Q_OFF + qs[0] * L::TILE, sbase + L::Q_OFF + qs[1] * L::TILE};
        for (int qt = 0; qt < (has1 ? 2 : 1) && ok; ++qt)
          ok = wait_bounded(&bar.q_full[qs[qt]], ((q_cnt + qt) / kQSlots) & 1, wc, 214);
        if (!ok) break;
        q_cnt += has1 ? 2 : 1;
        // Prologue: S of block 0 for both tiles.
        {
          const int s = kv_use % kStages;
          if (!wait_bounded(&bar.k_full[s], (kv_use / kStages) & 1, wc, 215)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int qt = 0; qt < 2; ++qt) {
            if (qt == 1 && !has1) break;
            mma_s<D>(tmem + L::s_col(qt), qa[qt], sbase + L::K_OFF + s * L::TILE, idesc_qk);
            umma_commit(&bar.s_full[qt]);
            if (n == 1) umma_commit(&bar.q_empty[qs[qt]]);   // this tile's last S
          }
          umma_commit(&bar.k_empty[s]);
        }
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t use = kv_use + j;
          const int s = use % kStages;
          const int s1 = (use + 1) % kStages;
          const bool more = j + 1 < n;
          if (!wait_bounded(&bar.v_full[s], (use / kStages) & 1, wc, 212)) { ok = false; break; }
          if (more && !wait_bounded(&bar.k_full[s1], ((use + 1) / kStages) & 1, wc, 216)) { ok = false; break; }
#pragma unroll
          for (int qt = 0; qt < 2; ++qt) {
            if (qt == 1 && !has1) break;
            const uint32_t o_tiles = qt ? o_tiles1 : o_tiles0;
            const uint32_t pv_cnt = qt ? pv_cnt1 : pv_cnt0;
            // The first P.V of a tile overwrites O: the previous tile's epilogue must have
            // read it out.
            if (j == 0 && o_tiles > 0 &&
                !wait_bounded(&bar.o_free[qt], (o_tiles - 1) & 1, wc, 213)) { ok = false; break; }
            if (!wait_bounded(&bar.p_full[qt], pv_cnt & 1, wc, 211)) { ok = false; break; }
            tc_fence_after();
            mma_pv<D>(tmem + L::o_col(qt), tmem + L::s_col(qt), sbase + L::V_OFF + s * L::TILE,
                      idesc_pv, j == 0);
            // The unit's last P.V is signalled for the epilogue; an earlier one needs no signal
            // of its own: S of the next block is issued after it, so s_full covers it.
            if (!more) umma_commit(&bar.pv_done[qt]);
            if (qt) ++pv_cnt1; else ++pv_cnt0;
            if (more) {   // after P_qt(j) was consumed (the tensor pipe runs in issue order)
              mma_s<D>(tmem + L::s_col(qt), qa[qt], sbase + L::K_OFF + s1 * L::TILE, idesc_qk);
              umma_commit(&bar.s_full[qt]);
              if (j + 2 == n) umma_commit(&bar.q_empty[qs[qt]]);   // this tile's last S
            }
          }
          if (!ok) break;
          umma_commit(&bar.v_empty[s]);
          if (more) umma_commit(&bar.k_empty[s1]);
        }
        kv_use += n;
        ++o_tiles0;
        if (has1) ++o_tiles1;
      }
      // Every issued MMA completes before TMEM is released.
      umma_commit(&bar.fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.fin, 0) && int64_t(global_timer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else {
    // ================================================================ softmax + epilogue
    const int qt = warp >> 2;                     // query tile of this warpgroup
    const int wq = warp & 3;                      // TMEM lane quadrant
    const int r = wq * 32 + lane;                 // row of the tile == TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t s_col = L::s_col(qt);
    const uint32_t o_col = L::o_col(qt);
    const int tok_in_tile = r / g;
    const int jh = r - tok_in_tile * g;
    uint32_t kv_use = 0, s_cnt = 0, pv_cnt = 0, split_seen = 0;
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Tile& tile = plan.tiles[t];
      const int n = tile_blocks(tile);
      const bool has1 = tile.qn > tpt;
      if (qt == 1 && !has1) {
        kv_use += n;
        if (tile.part >= 0 &&
            split_unit_complete(plan.counters, tile, &bar.merge_in, &bar.merge_out, &bar.merge_flag,
                                split_seen++, false, lane, wc, &ok))
          merge_unit<D>(tile, geo, p.part_o, p.part_lse, p.out);
        continue;
      }
      const int tok = qt * tpt + tok_in_tile;     // token index within the work tile
      const bool row_ok = tok < tile.qn && r < tpt * g;
      const int q_tok = tile.q0 + tok;
      const int head = tile.kv_head * g + jh;
      const int urow = tok * g + jh;               // row within the unit (partials)
      // A warp whose 32 rows are all padding does no softmax or epilogue work; it only keeps
      // in step with the barriers (and zeroes stale V rows when it belongs to the first tile).
      const bool live = __any_sync(0xffffffffu, row_ok);
      // Keys visible to this row, as a limit on the logical key index.
      int lim = tile.kv1;
      if (p.paged && plan.block_size > 0) {
        // causal plan: this query is token kv_len - qlen + i of its sequence
        const int qlen = plan.a[tile.req + 1] - plan.a[tile.req];
        lim = min(lim, plan.b[tile.req] - qlen + (q_tok - plan.a[tile.req]) + 1);
      } else if (!p.paged) {
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
      for (int j = 0; j < n; ++j) {
        const uint32_t use = kv_use + j;
        ok = __all_sync(0xffffffffu, wait_bounded(&bar.s_full[qt], s_cnt & 1, wc, 221));
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        const int key0 = tile.kv0 + j * kTcBlockKeys;
        const int nv = max(0, min(kTcBlockKeys, lim - key0));
        if (live) {
        // Row maximum of the raw scores with independent partial maxima (no serial chain);
        // keys past the row's limit become -inf (only in blocks that have any).
        const bool full = __all_sync(0xffffffffu, nv == kTcBlockKeys);
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + s_col + c * 32, sv[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_ld(sv[c]);
        if (!full) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c * 32 + e >= nv) sv[c][e] = __float_as_uint(-INFINITY);
        }
        float pm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) pm[e & 7] = fmaxf(pm[e & 7], __uint_as_float(sv[c][e]));
        const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                               fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) * p.scale_log2;
        const float mn = fmaxf(m, mx);
        // Keep the old maximum unless the new one exceeds it by 2^8 (exact after division).
        const bool need = (j == 0) || (mn > m + 8.f);
        const bool rescale = j > 0 && need && m != -INFINITY;
        const float corr = rescale ? fast_exp2(m - mn) : 1.f;
        if (need) m = mn;
        const float nbase = (m == -INFINITY) ? 0.f : -m;
        // p = 2^(s * scale - m), stored as bf16 over the first 64 columns of S; the row sum
        // adds the fp32 values (the bf16 rounding of P is unbiased and averages out).
        const uint64_t scale2 = f32x2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nbase2 = f32x2_pack(nbase, nbase);
        uint64_t ps[2] = {0, 0};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(sv[c][2 * e]), __uint_as_float(sv[c][2 * e + 1])),
                                         scale2, nbase2);
            const float p0 = fast_exp2(f32x2_lo(x)), p1 = fast_exp2(f32x2_hi(x));
            pk[e] = pack_bf16x2(p0, p1);
            ps[e & 1] = f32x2_add(ps[e & 1], f32x2_pack(p0, p1));
          }
          tmem_st16(lane_addr + s_col + c * 16, pk);
        }
        const float psum = f32x2_sum(ps[0]) + f32x2_sum(ps[1]);
        l = l * corr + psum;
        if (__any_sync(0xffffffffu, rescale)) {
          // O holds the sum through block j-1: P.V of block j-1 was issued before S of block
          // j, whose completion (s_full, waited for above) covers it.
          rescale_o<D>(lane_addr + o_col, corr);
        }
        tmem_wait_st();
        }
        // V rows past the block's valid keys hold stale or junk data: zero them (the first
        // tile's warpgroup does it; P.V of either tile is issued after its p_full).
        const int vb = min(kTcBlockKeys, tile.kv1 - key0);
        if (qt == 0 && r >= vb) {
          const int s = use % kStages;
          if (wait_bounded(&bar.v_full[s], (use / kStages) & 1, wc, 223)) {
            uint8_t* vrow = smem + L::V_OFF + s * L::TILE + r * 128;
#pragma unroll
            for (int c = 0; c < L::CH; ++c)
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(vrow + c * kChunkBytes + u * 16) = make_uint4(0, 0, 0, 0);
            fence_proxy_async_smem();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full[qt]);
      }
      if (!ok) break;
      kv_use += n;
      // ---------------------------------------------------------------- epilogue
      const bool split = tile.part >= 0;
      // pv_done completes once per unit of this tile (after its last P.V).
      if (!live) {
        if (n > 0) ++pv_cnt;
      } else {
      if (n > 0) {
        ok = __all_sync(0xffffffffu, wait_bounded(&bar.pv_done[qt], pv_cnt & 1, wc, 224));
        if (!ok) break;
        ++pv_cnt;
        tc_fence_after();
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (n > 0) {
          tmem_ld32(lane_addr + o_col + c * 32, ov);
          tmem_wait_ld(ov);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0u;
        }
        if (!row_ok) continue;
        // A thread writes its own row: with 32-byte stores every store fills whole sectors
        // (the rows of a warp are Hq * d elements apart).
        if (!split) {
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pkd[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
          __nv_bfloat16* row = p.out + (int64_t(q_tok) * geo.hq + head) * D + c * 32;
          if (p.wide_stores) {
#pragma unroll
            for (int e = 0; e < 2; ++e)
              st_global_v8(row + 16 * e, pkd[8 * e], pkd[8 * e + 1], pkd[8 * e + 2], pkd[8 * e + 3],
                           pkd[8 * e + 4], pkd[8 * e + 5], pkd[8 * e + 6], pkd[8 * e + 7]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(row);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * inv);
          float* row = p.part_o + int64_t(tile.part + urow) * D + c * 32;
          if (p.wide_stores) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              st_global_v8(row + 8 * e, ov[8 * e], ov[8 * e + 1], ov[8 * e + 2], ov[8 * e + 3], ov[8 * e + 4],
                           ov[8 * e + 5], ov[8 * e + 6], ov[8 * e + 7]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(row);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = make_uint4(ov[4 * e], ov[4 * e + 1], ov[4 * e + 2], ov[4 * e + 3]);
          }
        }
      }
      if (split && row_ok) p.part_lse[tile.part + urow] = l > 0.f ? m + fast_log2(l) : -INFINITY;
      }
      if (n > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.o_free[qt]);
      }
      // The CTA that completes the unit's last split merges its rows.
      if (split &&
          split_unit_complete(plan.counters, tile, &bar.merge_in, &bar.merge_out, &bar.merge_flag,
                              split_seen++, threadIdx.x == 0, lane, wc, &ok))
        merge_unit<D>(tile, geo, p.part_o, p.part_lse, p.out);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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
  prm.wide_stores = ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(part_o)) & 31) == 0;
  prm.timeout_ns = timeout_ns;
  cudaError_t e;
  if (geo.d == 128) {
    e = cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TcLayout<128>::SMEM);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attn_tc_kernel<128>, dim3(uint32_t(plan.num_ctas)), dim3(kTcThreads),
                   TcLayout<128>::SMEM, stream, prm);
  } else {
    e = cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TcLayout<64>::SMEM);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attn_tc_kernel<64>, dim3(uint32_t(plan.num_ctas)), dim3(kTcThreads),
                   TcLayout<64>::SMEM, stream, prm);
  }
  return e;
}

}  // namespace rae
