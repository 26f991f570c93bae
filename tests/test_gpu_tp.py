"""Tensor-parallel head sharding on the GPU (page "mstar.model.components.distributed.attention",
ParallelAttention): the o_proj partial kernel against a float64 matmul, and N ranks emulated
one after another on one GPU -- each with its own context, pools and plan for its head slice
-- whose partials, summed, equal the oracle's unsharded layer.  Only the sum stands in for the
all-reduce (the two-rank all-reduce itself is tested with gloo in test_tp.py).
"""
import numpy as np
import pytest
import torch

import oracle
from ragged_attention_encoder_b200 import Context, inputs
from ragged_attention_encoder_b200.tp import (TensorParallelCrossAttention, shard_heads,
                                              shard_w_o)

from gpu_util import assert_close, oracle_pools

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,hq,d,n,bias", [(1, 20, 64, 1280, True), (64, 5, 64, 1280, True),
                                           (130, 8, 128, 384, False), (257, 4, 64, 128, True),
                                           (2064, 8, 128, 4096, True)])
def test_o_proj_partial_matches_float64(m, hq, d, n, bias):
    g = torch.Generator(device="cuda").manual_seed(m + n)
    k = hq * d
    attn = torch.randn(m, hq, d, generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn(n, k, generator=g, device="cuda") / k ** 0.5).to(torch.bfloat16)
    b = torch.randn(n, generator=g, device="cuda").to(torch.bfloat16) if bias else None
    ctx = Context(hq, hq, d, 16)
    out = ctx.o_proj_partial(attn, w, b)
    torch.cuda.synchronize()
    ctx.check_device_status()
    ref = attn.reshape(m, k).double() @ w.double().T
    if bias:
        ref = ref + b.double()
    got = out.double()
    # fp32 accumulation of bf16 products: relative error of order k * 2^-24
    err = (got - ref).abs().max().item()
    rel = ((got - ref).norm() / ref.norm()).item()
    assert err <= 1e-3 and rel <= 1e-5, (err, rel)


def _shapes():
    # (seed, q_lens, ctx_lens, hq, hkv, d, P, world, hidden)
    return [
        (601, [1] * 6, [1500, 700, 33, 1, 900, 1200], 20, 20, 64, 16, 4, 1280),   # decode kernel
        (602, [7, 40, 1, 64], [300, 1000, 77, 2048], 32, 8, 128, 16, 2, 1024),    # 128-row tiles
        (603, [4, 4, 4], [4000, 9000, 130], 64, 8, 128, 64, 4, 512),               # swapped kernel
    ]


@pytest.mark.parametrize("seed,q_lens,ctx_lens,hq,hkv,d,P,world,hidden", _shapes())
def test_emulated_ranks_sum_to_the_unsharded_layer(seed, q_lens, ctx_lens, hq, hkv, d, P, world,
                                                   hidden):
    case = inputs.paged_case(seed, q_lens=q_lens, ctx_lens=ctx_lens, num_qo_heads=hq,
                             num_kv_heads=hkv, head_dim=d, page_size=P)
    g = torch.Generator().manual_seed(seed + 1)
    w_o = (torch.randn(hidden, hq * d, generator=g) / (hq * d) ** 0.5).to(torch.bfloat16)
    b_o = torch.randn(hidden, generator=g).to(torch.bfloat16)
    total = None
    for r in range(world):
        tp = TensorParallelCrossAttention(hq, hkv, d, P, rank=r, world=world)
        s = tp.shard
        kp = inputs.nan_pool(case.num_pages, s.num_kv_heads, P, d, "cuda")
        vp = inputs.nan_pool(case.num_pages, s.num_kv_heads, P, d, "cuda")
        tp.write_context(shard_heads(case.k_ctx, s.kv0, s.num_kv_heads).cuda(),
                         shard_heads(case.v_ctx, s.kv0, s.num_kv_heads).cuda(), case.cu_enc,
                         case.kv_page_indptr, case.kv_page_indices, kp, vp)
        plan = tp.plan(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices, case.kv_len,
                       case.num_pages)
        attn = tp.run(plan, shard_heads(case.q, s.q0, s.num_qo_heads).cuda(), kp, vp)
        # this rank's partial; the sum below stands in for the group's all-reduce
        part = tp.o_proj(attn, shard_w_o(w_o, s, d).cuda(), b_o.cuda(), reduce=False)
        torch.cuda.synchronize()
        tp.ctx.check_device_status()
        total = part if total is None else total + part
    kp, vp = oracle_pools(case)
    attn = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    ref = attn.reshape(attn.shape[0], -1) @ w_o.double().numpy().T + b_o.double().numpy()
    assert_close(total, ref, what=f"tp world {world}")
