// Context write: scatters packed encoder K/V [sum_enc, Hkv, d] into the paged pools
// [num_pages, Hkv, P, d] (M* page "mstar.engine.resources.attn.cross": the encode step writes
// the context once as an ordinary KV stream; later steps only read it).
//
// One CTA copies one page's worth of tokens for K and for V.  The source rows of a page are
// one contiguous block of ntok * Hkv * d elements, the destination is the page's Hkv runs of
// ntok * d elements, so both sides move in whole 16-byte vectors with coalesced accesses.
// HBM bound: algorithmic bytes = 2 (K and V) x 2 (read + write) x tokens x Hkv x d x 2 B.
#include "kernels.h"

namespace rae {
namespace {

__global__ void __launch_bounds__(256) context_write_kernel(const WriteItem* __restrict__ items,
                                                            const uint4* __restrict__ k_src,
                                                            const uint4* __restrict__ v_src,
                                                            uint4* __restrict__ k_pool,
                                                            uint4* __restrict__ v_pool,
                                                            int32_t hkv, int32_t vec_per_row,
                                                            int32_t page_size) {
  const WriteItem it = items[blockIdx.x];
  const int32_t per_tok = hkv * vec_per_row;          // 16-byte vectors per token (all heads)
  const int32_t n = it.ntok * per_tok;
  const int64_t src0 = int64_t(it.src_row) * per_tok;
  const int64_t page0 = int64_t(it.page) * hkv * page_size * vec_per_row;
  for (int32_t e = threadIdx.x; e < n; e += blockDim.x) {
    const int32_t slot = e / per_tok;
    const int32_t rem = e - slot * per_tok;
    const int32_t h = rem / vec_per_row;
    const int32_t u = rem - h * vec_per_row;
    const int64_t dst = page0 + (int64_t(h) * page_size + slot) * vec_per_row + u;
    const uint4 kv = __ldcs(k_src + src0 + e);   // streamed once
    const uint4 vv = __ldcs(v_src + src0 + e);
    k_pool[dst] = kv;
    v_pool[dst] = vv;
  }
}

}  // namespace

cudaError_t launch_context_write(const WriteItem* items, int64_t num_items, const void* k_src,
                                 const void* v_src, void* k_pool, void* v_pool,
                                 const Geometry& geo, cudaStream_t stream) {
  if (num_items == 0) return cudaSuccess;
  context_write_kernel<<<dim3(uint32_t(num_items)), 256, 0, stream>>>(
      items, static_cast<const uint4*>(k_src), static_cast<const uint4*>(v_src),
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), geo.hkv, geo.d / 8,
      geo.page_size);
  return cudaGetLastError();
}

}  // namespace rae
