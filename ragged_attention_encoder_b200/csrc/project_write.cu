// Fused K/V projection and context write (the encode step).
//
// M* page "mstar.model.components.attention" (CrossAttention.compute_kv): the encoder states
// [enc_len, hidden] go through the K and V linears (nn.Linear layout, weight [out, in]; the
// default has v biased and k not) into (enc_len, heads, head_dim) each.  Page
// "mstar.engine.resources.attn.cross": those K/V are the context, written once into the paged
// cache.  One kernel does both: a tcgen05 GEMM per 128-token x 256-column tile of [K | V],
// and an epilogue that adds the bias, rounds to bf16 and stores each token's row straight
// into its page slot, so the projected K/V never make a round trip through HBM.
//
// A tile's columns lie all in K or all in V (Hkv*d % 256 == 0; 128-column tiles with a
// 3-stage ring when only Hkv*d % 128 == 0).  The hidden dimension streams in 64-wide chunks
// through a TMA ring (A: hidden states, B: weight rows, both K-major with 128-byte swizzle)
// into S += A.B^T on the tensor core (one M=128 x N=tile MMA per 16-wide step), fp32 in TMEM.
// Warps: 0 TMA producer, 1 MMA issuer and TMEM owner, 2-5 epilogue (TMEM lane quadrant =
// warp % 4, one token row per thread).  Two CTAs fit on an SM, so one's epilogue overlaps
// the other's MMAs.  The grid runs the column tiles of a row block back to back,
// so each block of hidden states is read from HBM once and then from L2.  Every wait is
// bounded.
#include "kernels.h"
#include "ptx.cuh"

// Tiles 256 columns wide (when Hkv*d allows) with a 2-stage ring: 97 KB of shared memory, so
// two CTAs share an SM and one's epilogue overlaps the other's MMAs (measured: 580 us for the
// Whisper-large encode step, against 689 us with 3 stages and one CTA per SM, and 665 us
// with 128-column tiles).
#ifndef PW_BN_WIDE
#define PW_BN_WIDE 256
#define PW_STAGES_WIDE 2
#endif

namespace rae {
namespace {

constexpr int kPwThreads = 192;
constexpr int kPwChunk = 128 * 128;              // bytes: 128 rows x 64 bf16

// BN output columns per tile (128 or 256), STAGES chunks of the hidden dimension in flight.
template <int BN, int STAGES>
struct PwCfg {
  static constexpr int B_BYTES = BN * 128;                   // BN weight rows x 64 bf16
  static constexpr int STAGE_BYTES = kPwChunk + B_BYTES;     // A and B
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;          // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = BN;
};

template <int STAGES>
struct PwBars {
  uint64_t full[STAGES], empty[STAGES], acc_full;
  uint32_t tmem_base;
  int abort;
};

struct PwParams {
  CUtensorMap a, bk, bv;              // hidden [M, H]; w_k, w_v [Hkv*d, H]
  const __nv_bfloat16* bias_k;        // [Hkv*d] or null
  const __nv_bfloat16* bias_v;
  const WriteItem* items;             // page copies, in token order
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  int* err;
  int64_t timeout_ns;
  int32_t num_items;
  int32_t m;                          // tokens (rows of A)
  int32_t kchunks;                    // H / 64
  int32_t n_half;                     // Hkv * d
  int32_t hkv, d, page_size;
  int32_t wide_stores;                // both pools 32-byte aligned: one whole sector per store
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kPwThreads) project_write_kernel(const __grid_constant__ PwParams p) {
  using C = PwCfg<BN, STAGES>;
  static_assert(sizeof(PwBars<STAGES>) <= 256, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PwBars<STAGES>& bar = *reinterpret_cast<PwBars<STAGES>*>(smem + C::BAR_OFF);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;                  // column of [K | V]
  const int m0 = blockIdx.y * 128;                 // first token of the tile
  const bool is_v = n0 >= p.n_half;
  const int nl = is_v ? n0 - p.n_half : n0;        // column within K or V

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    mbar_init(&bar.acc_full, 1);
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.a);
    prefetch_tmap(is_v ? &p.bv : &p.bk);
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
      const CUtensorMap* mb = is_v ? &p.bv : &p.bk;
      const uint64_t pol = policy_evict_last();    // both operands are read by other CTAs
      int kc = 0;
      for (; kc < p.kchunks; ++kc) {
        const int s = kc % STAGES;
        if (kc >= STAGES && !wait_bounded(&bar.empty[s], ((kc / STAGES) - 1) & 1, wc, 501))
          break;
        mbar_arrive_expect_tx(&bar.full[s], uint32_t(C::STAGE_BYTES));
        tma_load_2d(smem + s * C::STAGE_BYTES, &p.a, &bar.full[s], kc * 64, m0, pol);
        tma_load_2d(smem + s * C::STAGE_BYTES + kPwChunk, mb, &bar.full[s], kc * 64, nl, pol);
      }
      // Every armed copy lands before the CTA may exit.
      for (int u = kc > STAGES ? kc - STAGES : 0; u < kc; ++u) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.full[u % STAGES], (u / STAGES) & 1) &&
               int64_t(global_timer_ns() - t0) < p.timeout_ns) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      for (int kc = 0; kc < p.kchunks; ++kc) {
        const int s = kc % STAGES;
        if (!wait_bounded(&bar.full[s], (kc / STAGES) & 1, wc, 502)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t b_addr = a_addr + kPwChunk;
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
    // Destination of this token: the write item that holds it (items ascend in token order).
    int64_t dst_row = -1;                          // (page * Hkv + 0) * P + slot
    if (m < p.m) {
      int lo = 0, hi = p.num_items - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.items[mid].src_row <= m) lo = mid; else hi = mid - 1;
      }
      const WriteItem it = p.items[lo];
      dst_row = int64_t(it.page) * p.hkv * p.page_size + it.slot0 + (m - it.src_row);
    }
    const bool ok = __all_sync(0xffffffffu, wait_bounded(&bar.acc_full, 0, wc, 503));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* pool = is_v ? p.v_pool : p.k_pool;
      const __nv_bfloat16* bias = is_v ? p.bias_v : p.bias_k;
      const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_addr + c * 32, v);
        tmem_wait_ld(v);
        if (dst_row < 0) continue;
        const int col = nl + c * 32;               // 32 columns inside one head
        const int h = col / p.d;
        const int e0 = col - h * p.d;
        uint32_t bw[16];
        if (bias) {
          const uint4* bp = reinterpret_cast<const uint4*>(bias + col);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 b4 = __ldg(bp + j);
            bw[4 * j] = b4.x;
            bw[4 * j + 1] = b4.y;
            bw[4 * j + 2] = b4.z;
            bw[4 * j + 3] = b4.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) bw[j] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]) + bf16lo_to_f32(bw[j]),
                              __uint_as_float(v[2 * j + 1]) + bf16hi_to_f32(bw[j]));
        // A thread's 64 bytes: with 32-byte stores each fills a whole sector (the rows of a
        // warp are d elements apart).
        __nv_bfloat16* row = pool + (dst_row + int64_t(h) * p.page_size) * p.d + e0;
        if (p.wide_stores) {
#pragma unroll
          for (int j = 0; j < 2; ++j)
            st_global_v8(row + 16 * j, pk[8 * j], pk[8 * j + 1], pk[8 * j + 2], pk[8 * j + 3], pk[8 * j + 4],
                         pk[8 * j + 5], pk[8 * j + 6], pk[8 * j + 7]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(row);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

namespace {

template <int BN, int STAGES>
cudaError_t launch_bn(const PwParams& prm, int m, cudaStream_t stream) {
  using C = PwCfg<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(project_write_kernel<BN, STAGES>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid(uint32_t(2 * prm.n_half / BN), uint32_t((m + 127) / 128));
  return launch_pdl(project_write_kernel<BN, STAGES>, grid, dim3(kPwThreads), size_t(C::SMEM),
                    stream, prm);
}

}  // namespace

int project_write_tile_cols(int n_half) { return n_half % 256 == 0 ? PW_BN_WIDE : 128; }

cudaError_t launch_project_write(const ProjectWriteArgs& a, cudaStream_t stream) {
  if (a.m == 0) return cudaSuccess;
  PwParams prm;
  prm.a = a.maps[0];
  prm.bk = a.maps[1];
  prm.bv = a.maps[2];
  prm.bias_k = static_cast<const __nv_bfloat16*>(a.bias_k);
  prm.bias_v = static_cast<const __nv_bfloat16*>(a.bias_v);
  prm.items = a.items;
  prm.k_pool = static_cast<__nv_bfloat16*>(a.k_pool);
  prm.v_pool = static_cast<__nv_bfloat16*>(a.v_pool);
  prm.err = a.err;
  prm.timeout_ns = a.timeout_ns;
  prm.num_items = int32_t(a.num_items);
  prm.m = a.m;
  prm.kchunks = a.hidden / 64;
  prm.n_half = a.geo.hkv * a.geo.d;
  prm.hkv = a.geo.hkv;
  prm.d = a.geo.d;
  prm.page_size = a.geo.page_size;
  prm.wide_stores = ((reinterpret_cast<uintptr_t>(a.k_pool) | reinterpret_cast<uintptr_t>(a.v_pool)) & 31) == 0;
  // (the weight maps' box height must be project_write_tile_cols(n_half))
  if (project_write_tile_cols(prm.n_half) != 128) return launch_bn<PW_BN_WIDE, PW_STAGES_WIDE>(prm, a.m, stream);
  return launch_bn<128, 3>(prm, a.m, stream);
}

}  // namespace rae
