// Split-KV merge, fused into the attention kernels.
//
// When the plan cuts a unit's keys over several tiles (so that every CTA of the persistent
// grid gets the same work), each split writes, per output row, its normalised fp32 partial
// O_i and lse_i = log2(sum_j 2^x_ij) (x = scaled score in log2 units).  The CTA that finishes
// a unit's last split -- found with one arrival counter per split unit -- merges the rows:
//     m = max_i lse_i,  w_i = 2^(lse_i - m),  O = sum_i w_i O_i / sum_i w_i
// summed in split order (deterministic whichever CTA merges) and written as bf16.  The
// counter is reset by that CTA, so the next run finds it at zero.
#pragma once
#include "kernels.h"
#include "ptx.cuh"

namespace rae {

// Called by every thread of the participating warps once their partial rows of a split tile
// are written.  `leader` is one thread of them.  Returns, in every participating thread,
// whether this CTA completed the unit (and must merge it).  bar_in counts one arrival per
// participating warp, bar_out one; `phase` counts the split tiles seen so far.
__device__ __forceinline__ bool split_unit_complete(int* counters, const Tile& tile, uint64_t* bar_in,
                                                    uint64_t* bar_out, volatile int* flag,
                                                    uint32_t phase, bool leader, int lane,
                                                    const WaitCtl& wc, bool* ok) {
  // The arrivals order every participating thread's partial stores before the leader's
  // device-scope fence (fences are cumulative), which orders them before the counter add.
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_in);
  if (leader) {
    int last = 0;
    if (wait_bounded(bar_in, phase & 1, wc, 301)) {
      __threadfence();
      const int old = atomicAdd(counters + tile.munit, 1);
      if (old == tile.nsplit - 1) {
        last = 1;
        counters[tile.munit] = 0;   // every split has arrived: ready for the next run
        __threadfence();            // the other splits' partials are read after this
      }
    }
    *flag = last;
    mbar_arrive(bar_out);
  }
  if (!wait_bounded(bar_out, phase & 1, wc, 302)) {
    *ok = false;
    return false;
  }
  return *flag != 0;   // partials are then read through L2 (ld.global.cg)
}

// Merges every row of the tile's unit; thread-strided over (row, 4-column group).
template <int D>
__device__ __forceinline__ void merge_split_unit(const Tile& tile, const Geometry& geo,
                                                 const float* part_o, const float* part_lse,
                                                 __nv_bfloat16* out, int tid, int nthreads) {
  constexpr int V = D / 4;
  const int rows = tile.qn * geo.g;
  const int base = tile.part - tile.split * rows;
  for (int e = tid; e < rows * V; e += nthreads) {
    const int r = e / V;
    const int c = e - r * V;
    float m = -INFINITY;
    for (int s = 0; s < tile.nsplit; ++s) m = fmaxf(m, __ldcg(part_lse + base + s * rows + r));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < tile.nsplit; ++s) {
        const int row = base + s * rows + r;
        const float w = fast_exp2(__ldcg(part_lse + row) - m);
        const float4 v = __ldcg(reinterpret_cast<const float4*>(part_o + int64_t(row) * D) + c);
        den += w;
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const int tok = tile.q0 + r / geo.g;
    const int head = tile.kv_head * geo.g + r % geo.g;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(out + (int64_t(tok) * geo.hq + head) * D + 4 * c) = pk;
  }
}

}  // namespace rae
