// Paged cross-attention for decode steps with few query rows per (request, KV head).
//
// M* page "mstar.engine.resources.attn.cross" (FlashInferCrossManager): non-causal attention
// of the decoder's packed queries over the context pages.  With one query token and a
// handful of heads per KV head there are at most 8 query rows per (request, KV head), about
// one multiply-add per byte of K/V read: HBM bound, far below the tensor-core ridge.  So this
// kernel runs on CUDA cores and spends its effort on keeping HBM busy:
//
//   * persistent CTAs walk the plan's tile list (balanced split-KV pieces);
//   * a producer warp streams 16-key chunks of K and V pages with cp.async.bulk into a
//     ring of shared-memory stages (4 chunks of K and 4 of V per stage, each chunk one
//     contiguous 16 x d run of a page), signalled by mbarrier transaction counts;
//   * four consumer warps each take one chunk per stage: scores with 16-byte vector reads,
//     reduced over the lanes that share a key with warp shuffles; online softmax in fp32
//     (scale folded into exp2); P.V accumulated in registers;
//   * at the end of a tile the four warps' (max, sum, O) are merged through shared memory
//     and the tile writes bf16 output, or an fp32 partial plus its log2-sum-exp when the
//     plan split the unit's keys.
#include "kernels.h"
#include "merge.cuh"
#include "ptx.cuh"

namespace rae {

#ifdef RAE_TEST_HOOKS
// Fault injection for the bounded-wait tests (test build only): the producer warp of this CTA
// arms no copies, so the CTA's consumer waits run out.  -1: off.
__device__ int g_silent_producer_cta = -1;
#endif

namespace {

constexpr int kSimtConsumers = 4;
constexpr int kSimtThreads = (kSimtConsumers + 1) * 32;

template <int D>
struct SimtCfg {
  static constexpr int CPL = D / 8;                 // 16-byte vectors per key row
  static constexpr int KPI = 32 / CPL;              // keys per warp-wide vector read
  static constexpr int ITERS = kSimtChunkKeys / KPI;
  static constexpr int CHUNK_ELEMS = kSimtChunkKeys * D;
  static constexpr int CHUNK_BYTES = CHUNK_ELEMS * 2;
  static constexpr int NST = D == 64 ? 6 : 3;       // stages in the ring
  static constexpr int STAGE_ELEMS = 2 * kSimtConsumers * CHUNK_ELEMS;   // K chunks, V chunks
};

template <int D, int R>
struct SimtSmem {
  using C = SimtCfg<D>;
  __nv_bfloat16 stage[C::NST][C::STAGE_ELEMS];
  float cm[kSimtConsumers][R];
  float cl[kSimtConsumers][R];
  float cacc[kSimtConsumers][R][D];
  uint64_t full[C::NST];
  uint64_t empty[C::NST];
  uint64_t merge_in, merge_out;   // split-unit arrival protocol
  int merge_flag;
  int abort;
};

template <int D, int R>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(
    DevPlan plan, Geometry geo, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k_pool, const __nv_bfloat16* __restrict__ v_pool,
    __nv_bfloat16* __restrict__ out, float* __restrict__ part_o, float* __restrict__ part_lse,
    int* err, float scale_log2, int64_t timeout_ns) {
  using C = SimtCfg<D>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  auto& sm = *reinterpret_cast<SimtSmem<D, R>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kSimtConsumers);
    }
    mbar_init(&sm.merge_in, kSimtConsumers);
    mbar_init(&sm.merge_out, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  const WaitCtl wc{&sm.abort, err, timeout_ns};

  const int t_begin = plan.cta_ptr[blockIdx.x];
  const int t_end = plan.cta_ptr[blockIdx.x + 1];

  if (warp == kSimtConsumers) {
    // ------------------------------------------------------------- producer warp
    // Lane i issues the copies of chunk i of a stage; each lane reads its chunk's page id
    // before the stage's empty-barrier wait, so those reads overlap it and each other.
    const uint64_t pol = policy_evict_first();
    uint32_t use = 0;
    bool ok = true;
#ifdef RAE_TEST_HOOKS
    if (int(blockIdx.x) == g_silent_producer_cta) ok = false;   // no copy is ever in flight
#endif
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Tile tile = plan.tiles[t];
      const int nch = (tile.kv1 - tile.kv0 + kSimtChunkKeys - 1) / kSimtChunkKeys;
      const int32_t* pages = plan.d + plan.c[tile.req];
      for (int c0 = 0; c0 < nch; c0 += kSimtConsumers, ++use) {
        const int s = use % C::NST;
        const int cnt = min(kSimtConsumers, nch - c0);
        int64_t row = 0;
        if (lane < cnt) {
          const int key = tile.kv0 + (c0 + lane) * kSimtChunkKeys;
          const int page = pages[key / geo.page_size];
          row = (int64_t(page) * geo.hkv + tile.kv_head) * geo.page_size + key % geo.page_size;
        }
        if (lane == 0 && use >= uint32_t(C::NST))
          ok = wait_bounded(&sm.empty[s], ((use / C::NST) - 1) & 1, wc, 101);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], uint32_t(cnt) * 2u * C::CHUNK_BYTES);
        __syncwarp();
        if (lane < cnt) {
          bulk_load(&sm.stage[s][lane * C::CHUNK_ELEMS], k_pool + row * D, C::CHUNK_BYTES,
                    &sm.full[s], pol);
          bulk_load(&sm.stage[s][(kSimtConsumers + lane) * C::CHUNK_ELEMS], v_pool + row * D,
                    C::CHUNK_BYTES, &sm.full[s], pol);
        }
      }
    }
    // Let every armed stage land before the CTA can exit (all of them when no wait gave up).
    if (lane == 0) {
      const uint32_t armed = use;
      for (uint32_t u = armed > uint32_t(C::NST) ? armed - C::NST : 0; u < armed; ++u) {
        const int s = u % C::NST;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&sm.full[s], (u / C::NST) & 1) &&
               int64_t(global_timer_ns() - t0) < timeout_ns) {
        }
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumer warps
  const int grp = lane / C::CPL;   // key within a warp-wide read
  const int cl = lane % C::CPL;    // 16-byte column of the key row
  uint32_t use = 0, split_seen = 0;
  for (int t = t_begin; t < t_end; ++t) {
    const Tile tile = plan.tiles[t];
    const int rows = tile.qn * geo.g;
    const int nch = (tile.kv1 - tile.kv0 + kSimtChunkKeys - 1) / kSimtChunkKeys;

    float qf[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < rows) {
        const int tok = tile.q0 + r / geo.g;
        const int head = tile.kv_head * geo.g + r % geo.g;
        const uint4 v = *reinterpret_cast<const uint4*>(q + (int64_t(tok) * geo.hq + head) * D + cl * 8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qf[r][2 * e] = bf16lo_to_f32(w[e]);
          qf[r][2 * e + 1] = bf16hi_to_f32(w[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[r][e] = 0.f;
      }
    }
    // Keys visible to each row: the tile's range, and under a causal plan (block_size 1) the
    // row's own position in its sequence (queries are the sequence's last tokens).
    int lim[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      lim[r] = tile.kv1;
      if (plan.block_size > 0 && r < rows) {
        const int q_first = plan.a[tile.req];
        const int qlen = plan.a[tile.req + 1] - q_first;
        const int tok = tile.q0 + r / geo.g;
        lim[r] = min(lim[r], plan.b[tile.req] - qlen + (tok - q_first) + 1);
      }
    }
    float m[R], l[R], acc[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      m[r] = -INFINITY;
      l[r] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
    }

    for (int c0 = 0; c0 < nch; c0 += kSimtConsumers, ++use) {
      const int s = use % C::NST;
      const bool ok = wait_bounded(&sm.full[s], (use / C::NST) & 1, wc, 102);
      const int chunk = c0 + warp;
      if (ok && chunk < nch) {
        const uint4* kc = reinterpret_cast<const uint4*>(&sm.stage[s][warp * C::CHUNK_ELEMS]);
        const uint4* vc =
            reinterpret_cast<const uint4*>(&sm.stage[s][(kSimtConsumers + warp) * C::CHUNK_ELEMS]);
        const int kbase = tile.kv0 + chunk * kSimtChunkKeys;
        float x[R][C::ITERS];
#pragma unroll
        for (int i = 0; i < C::ITERS; ++i) {
          const uint4 kv = kc[i * 32 + lane];
          const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
          float kf[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kf[2 * e] = bf16lo_to_f32(w[e]);
            kf[2 * e + 1] = bf16hi_to_f32(w[e]);
          }
          const int key = kbase + i * C::KPI + grp;
#pragma unroll
          for (int r = 0; r < R; ++r) {
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) dot = fmaf(qf[r][e], kf[e], dot);
#pragma unroll
            for (int o = C::CPL / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            x[r][i] = key < lim[r] ? dot * scale_log2 : -INFINITY;
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float cmax = x[r][0];
#pragma unroll
          for (int i = 1; i < C::ITERS; ++i) cmax = fmaxf(cmax, x[r][i]);
#pragma unroll
          for (int o = C::CPL; o < 32; o <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
          const float mn = fmaxf(m[r], cmax);
          if (mn == -INFINITY) {
#pragma unroll
            for (int i = 0; i < C::ITERS; ++i) x[r][i] = 0.f;   // nothing visible yet
            continue;
          }
          const float corr = fast_exp2(m[r] - mn);   // 0 when m was -inf
          m[r] = mn;
          float lsum = 0.f;
#pragma unroll
          for (int i = 0; i < C::ITERS; ++i) {
            x[r][i] = fast_exp2(x[r][i] - mn);          // 0 for masked keys
            lsum += x[r][i];
          }
          l[r] = l[r] * corr + lsum;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[r][e] *= corr;
        }
#pragma unroll
        for (int i = 0; i < C::ITERS; ++i) {
          if (kbase + i * C::KPI + grp >= tile.kv1) continue;   // V past the context may be junk
          const uint4 vv = vc[i * 32 + lane];
          const uint32_t w[4] = {vv.x, vv.y, vv.z, vv.w};
          float vf[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            vf[2 * e] = bf16lo_to_f32(w[e]);
            vf[2 * e + 1] = bf16hi_to_f32(w[e]);
          }
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(x[r][i], vf[e], acc[r][e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }

    // Sum the lanes that hold different keys of the same column.
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int o = C::CPL; o < 32; o <<= 1) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], o);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] += __shfl_xor_sync(0xffffffffu, acc[r][e], o);
      }
    }
    if (grp == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.cacc[warp][r][cl * 8 + e] = acc[r][e];
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        sm.cm[warp][r] = m[r];
        sm.cl[warp][r] = l[r];
      }
    }
    named_bar_sync(1, kSimtConsumers * 32);
    if (!sm.abort) {
      for (int e = threadIdx.x; e < rows * D; e += kSimtConsumers * 32) {
        const int r = e / D;
        const int dc = e - r * D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kSimtConsumers; ++w) mx = fmaxf(mx, sm.cm[w][r]);
        float num = 0.f, den = 0.f;
        if (mx != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kSimtConsumers; ++w) {
            const float f = fast_exp2(sm.cm[w][r] - mx);
            num += f * sm.cacc[w][r][dc];
            den += f * sm.cl[w][r];
          }
        }
        const float o = den > 0.f ? num / den : 0.f;
        if (tile.part < 0) {
          const int tok = tile.q0 + r / geo.g;
          const int head = tile.kv_head * geo.g + r % geo.g;
          out[(int64_t(tok) * geo.hq + head) * D + dc] = __float2bfloat16_rn(o);
        } else {
          part_o[int64_t(tile.part + r) * D + dc] = o;
          if (dc == 0) part_lse[tile.part + r] = den > 0.f ? mx + fast_log2(den) : -INFINITY;
        }
      }
    }
    if (tile.part >= 0) {
      // The CTA that completes the unit's last split merges its rows.
      bool ok = true;
      const bool last = split_unit_complete(plan.counters, tile, &sm.merge_in, &sm.merge_out,
                                            &sm.merge_flag, split_seen++, threadIdx.x == 0, lane,
                                            wc, &ok);
      if (last && !sm.abort)
        merge_split_unit<D, 32 / (D / 4)>(tile, geo, part_o, part_lse, out, threadIdx.x, kSimtConsumers * 32);
    }
    named_bar_sync(1, kSimtConsumers * 32);
  }
}

template <int D, int R>
cudaError_t launch_t(const DevPlan& plan, const Geometry& geo, const void* q, const void* k_pool,
                     const void* v_pool, void* out, float* part_o, float* part_lse, int* err,
                     float scale_log2, int64_t timeout_ns, cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem<D, R>);
  auto kern = decode_simt_kernel<D, R>;
  static bool attr_set = false;   // per template instance; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(kern, dim3(uint32_t(plan.num_ctas)), dim3(kSimtThreads), smem, stream, plan,
                    geo, static_cast<const __nv_bfloat16*>(q),
                    static_cast<const __nv_bfloat16*>(k_pool),
                    static_cast<const __nv_bfloat16*>(v_pool), static_cast<__nv_bfloat16*>(out),
                    part_o, part_lse, err, scale_log2, timeout_ns);
}

template <int D>
cudaError_t launch_d(const DevPlan& plan, const Geometry& geo, const void* q, const void* k_pool,
                     const void* v_pool, void* out, float* part_o, float* part_lse, int* err,
                     float scale_log2, int64_t timeout_ns, int rows_max, cudaStream_t stream) {
  if (rows_max <= 1)
    return launch_t<D, 1>(plan, geo, q, k_pool, v_pool, out, part_o, part_lse, err, scale_log2, timeout_ns, stream);
  if (rows_max <= 2)
    return launch_t<D, 2>(plan, geo, q, k_pool, v_pool, out, part_o, part_lse, err, scale_log2, timeout_ns, stream);
  if (rows_max <= 4)
    return launch_t<D, 4>(plan, geo, q, k_pool, v_pool, out, part_o, part_lse, err, scale_log2, timeout_ns, stream);
  return launch_t<D, 8>(plan, geo, q, k_pool, v_pool, out, part_o, part_lse, err, scale_log2, timeout_ns, stream);
}

}  // namespace

cudaError_t launch_decode_simt(const DevPlan& plan, const Geometry& geo, const void* q,
                               const void* k_pool, const void* v_pool, void* out,
                               float* part_o, float* part_lse, int* err, float scale_log2,
                               int64_t timeout_ns, int rows_max, cudaStream_t stream) {
  if (plan.num_ctas == 0) return cudaSuccess;
  if (geo.d == 128)
    return launch_d<128>(plan, geo, q, k_pool, v_pool, out, part_o, part_lse, err, scale_log2,
                         timeout_ns, rows_max, stream);
  return launch_d<64>(plan, geo, q, k_pool, v_pool, out, part_o, part_lse, err, scale_log2,
                      timeout_ns, rows_max, stream);
}

}  // namespace rae

#ifdef RAE_TEST_HOOKS
#include "rae_test_hooks.h"

extern "C" int rae_test_silence_producer(int32_t cta) {
  const int v = cta;
  return cudaMemcpyToSymbol(rae::g_silent_producer_cta, &v, sizeof(int)) == cudaSuccess
             ? RAE_OK
             : RAE_ERR_CUDA;
}
#endif
