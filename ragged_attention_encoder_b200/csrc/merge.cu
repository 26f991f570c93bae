// Split-KV merge.  A unit whose keys were split over several tiles left, per split i and
// output row, a normalised fp32 partial O_i and lse_i = log2(sum_j 2^(x_ij)) (x = scaled
// score in log2 units).  The merged row is
//     m = max_i lse_i,  w_i = 2^(lse_i - m),  O = sum_i w_i O_i / sum_i w_i
// accumulated in split order (deterministic; no atomics).  One warp per output row; the
// partials of a row are read once (HBM/L2 bound, a few MB at most).
#include "kernels.h"
#include "ptx.cuh"

namespace rae {
namespace {

template <int D>
__global__ void __launch_bounds__(128) merge_kernel(const MergeRow* __restrict__ rows,
                                                    int32_t num_rows,
                                                    const float* __restrict__ part_o,
                                                    const float* __restrict__ part_lse,
                                                    __nv_bfloat16* __restrict__ out) {
  constexpr int E = D / 32;   // elements per lane
  const int warp = int(blockIdx.x) * 4 + int(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= num_rows) return;
  const MergeRow mr = rows[warp];
  float m = -INFINITY;
  for (int s = 0; s < mr.nsplit; ++s) m = fmaxf(m, part_lse[mr.part0 + s * mr.stride]);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < mr.nsplit; ++s) {
      const int64_t row = int64_t(mr.part0) + int64_t(s) * mr.stride;
      const float w = fast_exp2(part_lse[row] - m);
      den += w;
      const float* src = part_o + row * D + lane * E;
      if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] += w * v.x;
        acc[1] += w * v.y;
        acc[2] += w * v.z;
        acc[3] += w * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] += w * v.x;
        acc[1] += w * v.y;
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* dst = out + int64_t(mr.out_row) * D + lane * E;
  if constexpr (E == 4) {
    uint2 pk;
    pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = pk;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
}

}  // namespace

cudaError_t launch_merge(const DevPlan& plan, const Geometry& geo, const float* part_o,
                         const float* part_lse, void* out, cudaStream_t stream) {
  if (plan.num_merge == 0) return cudaSuccess;
  const dim3 grid(uint32_t((plan.num_merge + 3) / 4));
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (geo.d == 128)
    merge_kernel<128><<<grid, 128, 0, stream>>>(plan.merge, plan.num_merge, part_o, part_lse, o);
  else
    merge_kernel<64><<<grid, 128, 0, stream>>>(plan.merge, plan.num_merge, part_o, part_lse, o);
  return cudaGetLastError();
}

}  // namespace rae
