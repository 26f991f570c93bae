// Launch interfaces of the CUDA kernels (internal to the library).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "plan.h"
#include "rae_internal.h"

namespace rae {

// Per-launch view of a plan image that sits in device memory.
struct DevPlan {
  const int32_t* cta_ptr;   // [num_ctas + 1]
  const Tile* tiles;        // [num_tiles]
  int* counters;            // arrival counter per split unit (zero between runs)
  const int32_t* a;         // paged: qo_indptr   ragged: cu_q
  const int32_t* b;         // paged: kv_len      ragged: cu_kv
  const int32_t* c;         // paged: kv_page_indptr
  const int32_t* d;         // paged: kv_page_indices
  int32_t num_ctas;
  int32_t block_size;
};

// Launches `kern` on `stream` with programmatic stream serialisation allowed: the kernel may
// be scheduled before the preceding kernel on the stream has finished (its prologue overlaps
// that kernel's tail) and calls griddep_wait before its first read of global memory.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

struct Geometry {
  int32_t hq, hkv, g, d, page_size;
};

// Context write: one CTA per page copy.
cudaError_t launch_context_write(const WriteItem* items, int64_t num_items, const void* k_src,
                                 const void* v_src, void* k_pool, void* v_pool,
                                 const Geometry& geo, cudaStream_t stream);

// Paged decode (<= 8 query rows per unit) on CUDA cores.
cudaError_t launch_decode_simt(const DevPlan& plan, const Geometry& geo, const void* q,
                               const void* k_pool, const void* v_pool, void* out,
                               float* part_o, float* part_lse, int* err, float scale_log2,
                               int64_t timeout_ns, int rows_max, cudaStream_t stream);

// tcgen05 attention over 128-row query tiles (paged or ragged K/V).
struct TcTensors {
  CUtensorMap q;   // 3D {d, Hq, total_q}, box {64, g, 128/g}
  CUtensorMap k;   // paged: 2D {d, pages*Hkv*P}, box {64, P}; ragged: 3D {d, Hkv, T}, box {64,1,128}
  CUtensorMap v;
};
cudaError_t launch_attn_tc(const DevPlan& plan, const Geometry& geo, bool paged,
                           const TcTensors& maps, void* out, float* part_o, float* part_lse,
                           int* err, float scale_log2, int64_t timeout_ns, cudaStream_t stream);

// tcgen05 attention with keys on the MMA M side, for n_rows (32 or 64) query rows, d = 128.
cudaError_t launch_attn_swapab(const DevPlan& plan, const Geometry& geo, int n_rows,
                               const TcTensors& maps, void* out, float* part_o, float* part_lse,
                               int* err, float scale_log2, int64_t timeout_ns, cudaStream_t stream);

// Fused K/V projection and context write: [K | V] = hidden . [w_k | w_v]^T (+ bias) on
// tcgen05, each token's row stored into its page slot.
struct ProjectWriteArgs {
  CUtensorMap maps[3];       // hidden {H, M} box {64, 128}; w_k, w_v {H, Hkv*d} box {64, tile cols}
  const void* bias_k;        // [Hkv*d] bf16 or null
  const void* bias_v;
  const WriteItem* items;    // device page copies, in token order
  int64_t num_items;
  void* k_pool;
  void* v_pool;
  int* err;
  int64_t timeout_ns;
  int32_t m;                 // tokens
  int32_t hidden;            // H, a multiple of 64
  Geometry geo;
};
cudaError_t launch_project_write(const ProjectWriteArgs& args, cudaStream_t stream);

// One tensor-parallel rank's o_proj partial: out [m, n] fp32 = attn [m, k] . w [n, k]^T
// (+ bias [n]); n % 128 == 0, k % 64 == 0.
struct OProjArgs {
  CUtensorMap maps[2];       // attn {k, m} box {64, 128}; w {k, n} box {64, 128}
  const void* bias;          // [n] bf16 or null
  void* out;                 // [m, n] fp32
  int* err;
  int64_t timeout_ns;
  int32_t m, n, k;
};
cudaError_t launch_o_proj(const OProjArgs& args, cudaStream_t stream);
int o_proj_tile_cols();

// Message of the calling thread's last failing context-free call (rae_write_context_noalloc).
const char* noalloc_last_error();
// Output columns per tile of the projection kernel (the weight maps' box height).
int project_write_tile_cols(int n_half);

}  // namespace rae
