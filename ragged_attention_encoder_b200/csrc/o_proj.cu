// Row-parallel output projection of one tensor-parallel rank.
//
// M* page "mstar.model.components.distributed.attention" (ParallelAttention): under tensor
// parallelism every rank holds the query and KV heads of its shard (KVConfig.shard narrows
// the head counts), runs attention on them, and applies its slice of o_proj: the rows of its
// heads' attention output [T, Hq_r * d] times its columns of W_o ([hidden, Hq_r * d] in
// nn.Linear layout).  The ranks' partials are then summed by one all-reduce, the only
// exchange of the layer.  This kernel computes one rank's partial
//     out[m, n] = sum_k attn[m, k] * w[n, k]  (+ bias[n] on the rank that adds it)
// in fp32, so that the sum over ranks rounds once.
//
// tcgen05 GEMM, one 128-token x 128-column tile per CTA: the k dimension streams in 64-wide
// chunks through a 4-stage TMA ring (A: attention rows, B: weight rows, both K-major with
// 128-byte swizzle) into fp32 accumulators in TMEM.  Warps: 0 TMA producer, 1 MMA issuer and
// TMEM owner, 2-5 epilogue (TMEM lane quadrant = warp % 4, one token row per thread, 32
// columns per TMEM load, written as eight 16-byte stores).  Rows past m are read as zeros by
// TMA and never stored.  Every wait is bounded.
#include "kernels.h"
#include "ptx.cuh"

namespace rae {
namespace {

constexpr int kOpThreads = 192;
constexpr int kOpBN = 128;
constexpr int kOpStages = 4;
constexpr int kOpChunk = 128 * 128;                       // 128 rows x 64 bf16
constexpr int kOpStageBytes = 2 * kOpChunk;               // A and B
constexpr int kOpBarOff = kOpStages * kOpStageBytes;
constexpr int kOpSmem = kOpBarOff + 256 + 1024;

struct OpBars {
  uint64_t full[kOpStages], empty[kOpStages], acc_full;
  uint32_t tmem_base;
  int abort;
};

struct OpParams {
  CUtensorMap a, b;            // attn [M, K]; w [N, K]
  const __nv_bfloat16* bias;   // [N] or null
  float* out;                  // [M, N]
  int* err;
  int64_t timeout_ns;
  int32_t m, n, kchunks;
};

__global__ void __launch_bounds__(kOpThreads) o_proj_kernel(const __grid_constant__ OpParams p) {
  static_assert(sizeof(OpBars) <= 256, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  OpBars& bar = *reinterpret_cast<OpBars*>(smem + kOpBarOff);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kOpBN;
  const int m0 = blockIdx.y * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    mbar_init(&bar.acc_full, 1);
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, kOpBN);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.a);
    prefetch_tmap(&p.b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t tmem = bar.tmem_base;
  const WaitCtl wc{&bar.abort, p.err, p.timeout_ns};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();   // both operands are read by other CTAs
      int kc = 0;
      for (; kc < p.kchunks; ++kc) {
        const int s = kc % kOpStages;
        if (kc >= kOpStages && !wait_bounded(&bar.empty[s], ((kc / kOpStages) - 1) & 1, wc, 601))
          break;
        mbar_arrive_expect_tx(&bar.full[s], uint32_t(kOpStageBytes));
        tma_load_2d(smem + s * kOpStageBytes, &p.a, &bar.full[s], kc * 64, m0, pol);
        tma_load_2d(smem + s * kOpStageBytes + kOpChunk, &p.b, &bar.full[s], kc * 64, n0, pol);
      }
      // Every armed copy lands before the CTA may exit.
      for (int u = kc > kOpStages ? kc - kOpStages : 0; u < kc; ++u) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.full[u % kOpStages], (u / kOpStages) & 1) &&
               int64_t(global_timer_ns() - t0) < p.timeout_ns) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kOpBN, false, false);
      for (int kc = 0; kc < p.kchunks; ++kc) {
        const int s = kc % kOpStages;
        if (!wait_bounded(&bar.full[s], (kc / kOpStages) & 1, wc, 602)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kOpStageBytes);
        const uint32_t b_addr = a_addr + kOpChunk;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_ss(tmem, smem_desc_sw128(a_addr + ks * 32, 16, 1024),
                  smem_desc_sw128(b_addr + ks * 32, 16, 1024), idesc, (kc > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&bar.empty[s]);
      }
      // Fires once every issued MMA has completed (also when a wait gave up).
      umma_commit(&bar.acc_full);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.acc_full, 0) && int64_t(global_timer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int wq = warp & 3;                       // TMEM lane quadrant
    const int r = wq * 32 + lane;                  // row of the tile == TMEM lane
    const int m = m0 + r;
    const bool ok = __all_sync(0xffffffffu, wait_bounded(&bar.acc_full, 0, wc, 603));
    if (ok) {
      tc_fence_after();
      const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
#pragma unroll
      for (int c = 0; c < kOpBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_addr + c * 32, v);
        tmem_wait_ld(v);
        if (m >= p.m) continue;
        const int col = n0 + c * 32;
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
        if (p.bias) {
          const uint4* bp = reinterpret_cast<const uint4*>(p.bias + col);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 b4 = __ldg(bp + j);
            const uint32_t bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              f[8 * j + 2 * e] += bf16lo_to_f32(bw[e]);
              f[8 * j + 2 * e + 1] += bf16hi_to_f32(bw[e]);
            }
          }
        }
        float4* dst = reinterpret_cast<float4*>(p.out + int64_t(m) * p.n + col);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kOpBN);
  }
}

}  // namespace

int o_proj_tile_cols() { return kOpBN; }

cudaError_t launch_o_proj(const OProjArgs& a, cudaStream_t stream) {
  if (a.m == 0 || a.n == 0) return cudaSuccess;
  OpParams prm;
  prm.a = a.maps[0];
  prm.b = a.maps[1];
  prm.bias = static_cast<const __nv_bfloat16*>(a.bias);
  prm.out = static_cast<float*>(a.out);
  prm.err = a.err;
  prm.timeout_ns = a.timeout_ns;
  prm.m = a.m;
  prm.n = a.n;
  prm.kchunks = a.k / 64;
  cudaError_t e = cudaFuncSetAttribute(o_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOpSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid(uint32_t(a.n / kOpBN), uint32_t((a.m + 127) / 128));
  return launch_pdl(o_proj_kernel, grid, dim3(kOpThreads), size_t(kOpSmem), stream, prm);
}

}  // namespace rae
