"""Tensor-parallel (head-sharded) cross-attention over several GPUs, one process per GPU.

M* page "mstar.model.components.distributed.attention" (ParallelAttention): the query, key
and value heads are split over the ranks of a tensor-parallel group -- KVConfig.shard narrows
the head counts to one rank's slice -- and the only exchange of the layer is the all-reduce
inside the row-parallel output projection.  Page "mstar.model.components.attention"
(CrossAttention) notes that the cross-attention there is not yet split over heads; this
module is that split for the cross-attention path of this library:

  * rank r of N owns KV heads [r * Hkv / N, (r + 1) * Hkv / N) and the g = Hq / Hkv query
    heads of each (whole GQA groups, so a query head and its KV head always live on the same
    rank and the head map h -> h // g holds inside every shard);
  * each rank keeps its own context pools (its heads only) under the same page table, plans
    with its local head counts and runs the unchanged kernels on its slice;
  * each rank multiplies its heads' attention output by its columns of W_o
    (``Context.o_proj_partial``, a tcgen05 GEMM with fp32 output; one rank adds the bias), and
    one all-reduce (torch.distributed; NCCL over NVLink on GPUs) sums the partials.

Everything here is host-side plumbing: the head partition, weight slicing and the collective
call.  The arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from .api import Context


@dataclass(frozen=True)
class HeadShard:
    """One rank's slice of the heads: KV heads [kv0, kv1), query heads [q0, q1)."""
    rank: int
    world: int
    kv0: int
    kv1: int
    q0: int
    q1: int

    @property
    def num_kv_heads(self) -> int:
        return self.kv1 - self.kv0

    @property
    def num_qo_heads(self) -> int:
        return self.q1 - self.q0


def head_shard(num_qo_heads: int, num_kv_heads: int, rank: int, world: int) -> HeadShard:
    """The contiguous slice of whole KV heads (and their query heads) that rank owns."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    if num_kv_heads <= 0 or num_qo_heads % num_kv_heads:
        raise ValueError("num_qo_heads must be a positive multiple of num_kv_heads")
    if num_kv_heads % world:
        raise ValueError(f"{num_kv_heads} KV heads do not split evenly over {world} ranks")
    g = num_qo_heads // num_kv_heads
    per = num_kv_heads // world
    kv0 = rank * per
    return HeadShard(rank, world, kv0, kv0 + per, kv0 * g, (kv0 + per) * g)


def shard_heads(x: torch.Tensor, first: int, count: int) -> torch.Tensor:
    """Heads [first, first + count) of a [tokens, heads, d] (or pool [pages, heads, P, d])
    tensor, as a contiguous copy: what a rank holds of a full-head tensor."""
    return x.narrow(1, first, count).contiguous()


def shard_w_o(w_o: torch.Tensor, shard: HeadShard, head_dim: int) -> torch.Tensor:
    """A rank's columns of W_o ([hidden, Hq * d], nn.Linear layout): the inputs that come
    from its query heads, [hidden, Hq_r * d], contiguous."""
    return w_o[:, shard.q0 * head_dim:shard.q1 * head_dim].contiguous()


class TensorParallelCrossAttention:
    """The cross-attention of one tensor-parallel rank: plan/run on its heads, then its o_proj
    partial and the group's all-reduce.

    ``rank``/``world`` place this process in the tensor-parallel group; ``group`` is the
    torch.distributed process group of the all-reduce (None: the default group).  Capacity
    keywords go to the rank's Context.
    """

    def __init__(self, num_qo_heads: int, num_kv_heads: int, head_dim: int, page_size: int = 16,
                 *, rank: int = 0, world: int = 1, group=None, device=None, **capacities):
        self.shard = head_shard(num_qo_heads, num_kv_heads, rank, world)
        self.head_dim = head_dim
        self.group = group
        self.ctx = Context(self.shard.num_qo_heads, self.shard.num_kv_heads, head_dim, page_size,
                           device=device, **capacities)

    # the rank's own context write, plan and run are the single-GPU calls on its heads
    def write_context(self, k_local, v_local, cu_enc, page_indptr, page_indices, k_pool, v_pool):
        self.ctx.write_context(k_local, v_local, cu_enc, page_indptr, page_indices, k_pool, v_pool)

    def plan(self, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages, **kw):
        return self.ctx.plan_paged(qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages,
                                   **kw)

    def run(self, plan, q_local, k_pool, v_pool, out=None):
        return self.ctx.run_paged(plan, q_local, k_pool, v_pool, out)

    def o_proj(self, attn_local, w_o_local, bias=None, out=None, reduce: bool = True):
        """Sum over the group of attn_local . w_o_local^T; ``bias`` is added by rank 0 only.
        With reduce=False this rank's partial is returned unreduced."""
        part = self.ctx.o_proj_partial(attn_local, w_o_local,
                                       bias if self.shard.rank == 0 else None, out)
        if reduce and self.shard.world > 1:
            import torch.distributed as dist
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
        return part

    def forward(self, plan, q_local, k_pool, v_pool, w_o_local, bias=None, attn_out=None,
                out=None):
        """One layer's cross-attention of this rank's heads followed by the reduced output
        projection: [tokens, hidden] fp32 on every rank."""
        attn = self.run(plan, q_local, k_pool, v_pool, attn_out)
        return self.o_proj(attn, w_o_local, bias, out)
