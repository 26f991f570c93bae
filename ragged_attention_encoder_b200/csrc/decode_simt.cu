// Paged cross-attention for decode steps with few query rows per (request, KV head).
//
// M* page "mstar.engine.resources.attn.cross" (FlashInferCrossManager): non-causal attention
// of the decoder's packed queries over the context pages.  With one query token and a
// handful of heads per KV head there are at most 8 query rows per (request, KV head), about
// one multiply-add per byte of K/V read: HBM bound, far below the tensor-core ridge.  So this
// kernel runs on CUDA cores and spends its effort on keeping HBM busy with long reads:
//
//   * persistent CTAs walk the plan's tile list (balanced split-KV pieces); a work unit is
//     (request, up to four adjacent KV heads, key range);
//   * a producer warp streams 16-key chunks of K and V with cp.async.bulk into a ring of
//     shared-memory stages.  A stage holds one chunk of every KV head of the unit.  With
//     16-token pages the chunk is a whole page, and the unit's heads are adjacent in the pool
//     [pages, Hkv, P, d], so each stage is ONE contiguous run of heads x 16 x d for K and one
//     for V (8 KB each at d = 64 and four heads, instead of four 2 KB runs); stages are
//     signalled by mbarrier transaction counts;
//   * consumer warp w owns KV head w of the unit for the whole key range: scores with 16-byte
//     vector reads, reduced over the lanes that share a key with warp shuffles; online
//     softmax in fp32 (scale folded into exp2); P.V accumulated in registers.  A warp sees
//     every key of its head, so no cross-warp merge is needed: each warp writes its rows as
//     bf16, or as an fp32 partial plus its log2-sum-exp when the plan split the unit's keys.
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

constexpr int kSimtConsumers = kSimtMaxHeads;   // one consumer warp per KV head of a unit
constexpr int kSimtThreads = (kSimtConsumers + 1) * 32;

template <int D>
struct SimtCfg {
  static constexpr int CPL = D / 8;                 // 16-byte vectors per key row
  static constexpr int KPI = 32 / CPL;              // keys per warp-wide vector read
  static constexpr int ITERS = kSimtChunkKeys / KPI;
  static constexpr int CHUNK_ELEMS = kSimtChunkKeys * D;
  static constexpr int CHUNK_BYTES = CHUNK_ELEMS * 2;
  // Stages in the ring: at d = 64 five 16 KB stages per CTA (two CTAs per SM) streamed
  // faster than four, six or seven.
  static constexpr int NST = D == 64 ? 5 : 3;
  static constexpr int STAGE_ELEMS = 2 * kSimtConsumers * CHUNK_ELEMS;   // K chunks, V chunks
};

template <int D>
struct SimtSmem {
  using C = SimtCfg<D>;
  __nv_bfloat16 stage[C::NST][C::STAGE_ELEMS];   // [K: head][16][d], then [V: head][16][d]
  uint64_t full[C::NST];
  uint64_t empty[C::NST];
  uint64_t merge_in, merge_out;   // split-unit arrival protocol
  int merge_flag;
  int abort;
};

template <int D, int R>
__global__ void __maxnreg__(200) decode_simt_kernel(
    DevPlan plan, Geometry geo, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k_pool, const __nv_bfloat16* __restrict__ v_pool,
    __nv_bfloat16* __restrict__ out, float* __restrict__ part_o, float* __restrict__ part_lse,
    int* err, float scale_log2, int64_t timeout_ns) {
  using C = SimtCfg<D>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  auto& sm = *reinterpret_cast<SimtSmem<D>*>(smem_raw);
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
  const int P = geo.page_size;

  if (warp == kSimtConsumers) {
    // ------------------------------------------------------------- producer warp
    // The page ids of 32 chunks at a time are read one per lane (the reads overlap each
    // other and the stage waits); lane 0 takes the waits and arms the transaction counts.
    // With P == 16 a stage is two copies (K and V, all heads of the unit); otherwise lanes
    // 0 .. nh-1 copy the heads' K chunks and lanes nh .. 2 nh - 1 their V chunks.
    const uint64_t pol = policy_evict_first();
    uint32_t use = 0;
    bool ok = true;
#ifdef RAE_TEST_HOOKS
    if (int(blockIdx.x) == g_silent_producer_cta) ok = false;   // no copy is ever in flight
#endif
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Tile tile = plan.tiles[t];
      const int nch = (tile.kv1 - tile.kv0 + kSimtChunkKeys - 1) / kSimtChunkKeys;
      const int nh = tile.nkvh;
      const int32_t* pages = plan.d + plan.c[tile.req];
      for (int c0 = 0; c0 < nch && ok; c0 += 32) {
        int my_page = 0;
        if (c0 + lane < nch) my_page = pages[(tile.kv0 + (c0 + lane) * kSimtChunkKeys) / P];
        const int cend = min(nch - c0, 32);
        for (int ci = 0; ci < cend; ++ci, ++use) {
          const int s = use % C::NST;
          const int page = __shfl_sync(0xffffffffu, my_page, ci);
          const int slot = (tile.kv0 + (c0 + ci) * kSimtChunkKeys) % P;
          if (lane == 0 && use >= uint32_t(C::NST))
            ok = wait_bounded(&sm.empty[s], ((use / C::NST) - 1) & 1, wc, 101);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], uint32_t(nh) * 2u * C::CHUNK_BYTES);
          __syncwarp();
          // first pool row of head tile.kv_head of this chunk
          const int64_t row0 = (int64_t(page) * geo.hkv + tile.kv_head) * P + slot;
          if (P == kSimtChunkKeys) {
            if (lane < 2)
              bulk_load(&sm.stage[s][lane * kSimtConsumers * C::CHUNK_ELEMS],
                        (lane == 0 ? k_pool : v_pool) + row0 * D, uint32_t(nh) * C::CHUNK_BYTES,
                        &sm.full[s], pol);
          } else if (lane < 2 * nh) {
            const int kv = lane >= nh;             // 0: K, 1: V
            const int h = lane - kv * nh;
            bulk_load(&sm.stage[s][(kv * kSimtConsumers + h) * C::CHUNK_ELEMS],
                      (kv ? v_pool : k_pool) + (row0 + int64_t(h) * P) * D, C::CHUNK_BYTES,
                      &sm.full[s], pol);
          }
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
    const bool active = warp < tile.nkvh;          // this warp's KV head is in the unit
    const int kvh = tile.kv_head + warp;
    const int rows = tile.qn * geo.g;              // rows of this warp's KV head
    const int hpt = tile.nkvh * geo.g;             // query heads per token in the unit
    const int nch = (tile.kv1 - tile.kv0 + kSimtChunkKeys - 1) / kSimtChunkKeys;

    float qf[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (active && r < rows) {
        const int tok = tile.q0 + r / geo.g;
        const int head = kvh * geo.g + r % geo.g;
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

    for (int c = 0; c < nch; ++c, ++use) {
      const int s = use % C::NST;
      const bool ok = wait_bounded(&sm.full[s], (use / C::NST) & 1, wc, 102);
      if (ok && active) {
        const uint4* kc = reinterpret_cast<const uint4*>(&sm.stage[s][warp * C::CHUNK_ELEMS]);
        const uint4* vc =
            reinterpret_cast<const uint4*>(&sm.stage[s][(kSimtConsumers + warp) * C::CHUNK_ELEMS]);
        const int kbase = tile.kv0 + c * kSimtChunkKeys;
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
    if (active && grp == 0 && !sm.abort) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r >= rows) break;
        const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
        const int tok = tile.q0 + r / geo.g;
        const int gi = r % geo.g;
        if (tile.part < 0) {
          uint4 pk;
          pk.x = pack_bf16x2(acc[r][0] * inv, acc[r][1] * inv);
          pk.y = pack_bf16x2(acc[r][2] * inv, acc[r][3] * inv);
          pk.z = pack_bf16x2(acc[r][4] * inv, acc[r][5] * inv);
          pk.w = pack_bf16x2(acc[r][6] * inv, acc[r][7] * inv);
          *reinterpret_cast<uint4*>(out + (int64_t(tok) * geo.hq + kvh * geo.g + gi) * D + cl * 8) = pk;
        } else {
          // unit row: (token, query head within the unit), token-major
          const int urow = (r / geo.g) * hpt + warp * geo.g + gi;
          float4* dst = reinterpret_cast<float4*>(part_o + int64_t(tile.part + urow) * D + cl * 8);
          dst[0] = make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
          dst[1] = make_float4(acc[r][4] * inv, acc[r][5] * inv, acc[r][6] * inv, acc[r][7] * inv);
          if (cl == 0)
            part_lse[tile.part + urow] = l[r] > 0.f ? m[r] + fast_log2(l[r]) : -INFINITY;
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
        merge_split_unit<D, 32 / (D / 4)>(tile, geo, tile.kv_head * geo.g, hpt, part_o, part_lse,
                                          out, threadIdx.x, kSimtConsumers * 32);
    }
  }
}

template <int D, int R>
cudaError_t launch_t(const DevPlan& plan, const Geometry& geo, const void* q, const void* k_pool,
                     const void* v_pool, void* out, float* part_o, float* part_lse, int* err,
                     float scale_log2, int64_t timeout_ns, cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem<D>);
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
