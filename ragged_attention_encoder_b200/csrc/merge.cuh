// Split-KV merge, fused into the attention kernels.
//
// When the plan cuts a unit's keys over several tiles (so that every CTA of the persistent
// grid gets the same work), each split writes, per output row, its normalised fp32 partial
// O_i and lse_i = log2(sum_j 2^x_ij) (x = scaled score in log2 units).  The CTA that finishes
// a unit's last split -- found with one arrival counter per split unit -- merges the rows:
//     m = max_i lse_i,  w_i = 2^(lse_i - m),  O = sum_i w_i O_i / sum_i w_i
// accumulated in split order with a running maximum (deterministic whichever CTA merges) and
// written as bf16.  The counter is reset by that CTA, so the next run finds it at zero.
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

// Merges every row of the tile's unit.  The participating threads are whole warps
// (tid = 32 * warp + lane, nthreads a multiple of 32).  A row's D/4 float4 column groups go to
// consecutive lanes (one row per warp for D = 128, two for D = 64), so every partial row is
// one coalesced read; each warp keeps kRows rows in flight (a multiple of the rows per warp
// pass) and combines the splits in one online pass (running maximum, rescaled sums), in
// split order.
//
// A unit's rows are (token, query head) pairs, token-major: row r is token tile.q0 + r / hpt,
// query head head0 + r % hpt, where hpt is the number of query heads per token in the unit
// (g for one KV head; g times the KV heads of the unit when it holds several).
template <int D, int kRows>
__device__ __forceinline__ void merge_split_unit(const Tile& tile, const Geometry& geo, int head0,
                                                 int hpt, const float* part_o,
                                                 const float* part_lse, __nv_bfloat16* out,
                                                 int tid, int nthreads) {
  constexpr int V = D / 4;              // float4 column groups per row
  constexpr int RPW = 32 / V;           // rows per warp and pass
  constexpr int U = kRows / RPW;        // passes unrolled
  static_assert(U >= 1 && U * RPW == kRows, "kRows must be a multiple of the rows per pass");
  const int rows = tile.qn * hpt;
  const int base = tile.part - tile.split * rows;
  const int ns = tile.nsplit;
  const int lane = tid & 31;
  const int c = lane % V;
  const int rsub = lane / V;
  for (int r0 = (tid >> 5) * kRows; r0 < rows; r0 += (nthreads >> 5) * kRows) {
    float m[U], den[U];
    float4 acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      m[u] = -INFINITY;
      den[u] = 0.f;
      acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int s = 0; s < ns; ++s) {
      float l[U];
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int r = r0 + u * RPW + rsub;
        l[u] = -INFINITY;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < rows) {
          const int row = base + s * rows + r;
          l[u] = __ldcg(part_lse + row);
          v[u] = __ldcg(reinterpret_cast<const float4*>(part_o + int64_t(row) * D) + c);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (l[u] == -INFINITY) continue;             // this split saw no key of the row
        const float mn = fmaxf(m[u], l[u]);
        const float a = fast_exp2(m[u] - mn);         // 0 while m is still -inf
        const float b = fast_exp2(l[u] - mn);
        acc[u].x = acc[u].x * a + v[u].x * b;
        acc[u].y = acc[u].y * a + v[u].y * b;
        acc[u].z = acc[u].z * a + v[u].z * b;
        acc[u].w = acc[u].w * a + v[u].w * b;
        den[u] = den[u] * a + b;
        m[u] = mn;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RPW + rsub;
      if (r >= rows) continue;
      const float inv = den[u] > 0.f ? 1.f / den[u] : 0.f;
      const int tok = tile.q0 + r / hpt;
      const int head = head0 + r % hpt;
      uint2 pk;
      pk.x = pack_bf16x2(acc[u].x * inv, acc[u].y * inv);
      pk.y = pack_bf16x2(acc[u].z * inv, acc[u].w * inv);
      *reinterpret_cast<uint2*>(out + (int64_t(tok) * geo.hq + head) * D + 4 * c) = pk;
    }
  }
}

}  // namespace rae
