"""Tensor-parallel head sharding (page "mstar.model.components.distributed.attention",
ParallelAttention; KVConfig.shard) on CPU: the partition of heads, per-rank plans, and -- with
two and four gloo ranks -- that the all-reduced o_proj partials of the ranks' head slices equal
the unsharded layer.  Each rank's attention is the float64 oracle here (no GPU); the GPU
kernels on the same slices are checked in test_gpu_tp.py.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from ragged_attention_encoder_b200 import inputs, plan_paged_host  # noqa: E402
from ragged_attention_encoder_b200.tp import head_shard, shard_heads, shard_w_o  # noqa: E402


@pytest.mark.parametrize("hq,hkv,world", [(20, 20, 4), (32, 8, 2), (32, 8, 8), (64, 8, 4),
                                          (4, 2, 2), (6, 3, 3)])
def test_shards_partition_whole_gqa_groups(hq, hkv, world):
    g = hq // hkv
    seen_q, seen_kv = [], []
    for r in range(world):
        s = head_shard(hq, hkv, r, world)
        assert s.num_kv_heads == hkv // world and s.num_qo_heads == hq // world
        seen_kv += list(range(s.kv0, s.kv1))
        seen_q += list(range(s.q0, s.q1))
        for h in range(s.q0, s.q1):                    # every query head's KV head is local
            assert s.kv0 <= h // g < s.kv1
    assert seen_kv == list(range(hkv)) and seen_q == list(range(hq))


def test_shards_reject_uneven_splits():
    with pytest.raises(ValueError):
        head_shard(20, 20, 0, 8)
    with pytest.raises(ValueError):
        head_shard(32, 8, 2, 2)
    with pytest.raises(ValueError):
        head_shard(30, 8, 0, 2)


def test_weight_slice_is_the_ranks_input_columns():
    w = torch.arange(6 * 24, dtype=torch.float64).reshape(6, 24)      # hidden 6, Hq 4 x d 6
    s = head_shard(4, 2, 1, 2)                                          # query heads 2, 3
    ws = shard_w_o(w, s, 6)
    assert ws.shape == (6, 12) and ws.is_contiguous()
    assert torch.equal(ws, w[:, 12:24])
    x = torch.arange(2 * 4 * 3).reshape(2, 4, 3)
    assert torch.equal(shard_heads(x, 1, 2), x[:, 1:3])


def test_rank_plans_cover_their_heads():
    """Each rank plans its slice with its local head counts from the same page table."""
    c = inputs.workload(3)
    for world in (2, 4):
        rows = 0
        for r in range(world):
            s = head_shard(c.num_qo_heads, c.num_kv_heads, r, world)
            p = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len,
                                c.num_pages, num_qo_heads=s.num_qo_heads,
                                num_kv_heads=s.num_kv_heads, head_dim=c.head_dim,
                                page_size=c.page_size, num_sms=148)
            t = p["tiles"]
            g = s.num_qo_heads // s.num_kv_heads
            assert int(t[:, 1].max()) < s.num_kv_heads          # local KV head indices
            # rows of the unsplit pieces plus one piece of every split unit
            first = t[t[:, 7] == 0]
            rows += int((first[:, 3] * g * first[:, 10]).sum())
        assert rows == int(c.qo_indptr[-1]) * c.num_qo_heads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_inputs(hidden=48):
    case = inputs.paged_case(501, q_lens=[1, 5, 2, 3], ctx_lens=[40, 100, 17, 64], num_qo_heads=8,
                             num_kv_heads=4, head_dim=16, page_size=16, pool_pages=24)
    g = torch.Generator().manual_seed(502)
    w_o = torch.randn(hidden, case.num_qo_heads * case.head_dim, generator=g, dtype=torch.float64)
    b_o = torch.randn(hidden, generator=g, dtype=torch.float64)
    return case, w_o, b_o


def _oracle_pools(case):
    import oracle
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    return oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                case.kv_page_indices, kp, vp)


def _rank_main(rank, world, port, swap, queue):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        case, w_o, b_o = _layer_inputs()
        s = head_shard(case.num_qo_heads, case.num_kv_heads, rank, world)
        kp, vp = _oracle_pools(case)
        # what this rank holds: its query heads, its KV heads' pools, its W_o columns
        q_l = shard_heads(case.q, s.q0, s.num_qo_heads)
        kp_l = shard_heads(kp, s.kv0, s.num_kv_heads)
        vp_l = shard_heads(vp, s.kv0, s.num_kv_heads)
        ws = shard_w_o(w_o, head_shard(case.num_qo_heads, case.num_kv_heads,
                                       (rank + 1) % world if swap else rank, world),
                       case.head_dim)
        attn = oracle.paged_cross_attention(q_l, kp_l, vp_l, case.qo_indptr, case.kv_page_indptr,
                                            case.kv_page_indices, case.kv_len)
        part = torch.from_numpy(attn.reshape(attn.shape[0], -1)) @ ws.T
        if rank == 0:
            part = part + b_o
        dist.all_reduce(part)
        queue.put((rank, part.numpy()))
    finally:
        dist.destroy_process_group()


def _run_ranks(world, swap=False):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, swap, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, part = queue.get(timeout=240)
        out[rank] = part
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def _unsharded():
    import oracle
    case, w_o, b_o = _layer_inputs()
    kp, vp = _oracle_pools(case)
    attn = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    return (torch.from_numpy(attn.reshape(attn.shape[0], -1)) @ w_o.T + b_o).numpy()


@pytest.mark.parametrize("world", [2, 4])
def test_all_reduced_partials_equal_the_unsharded_layer(world):
    ref = _unsharded()
    out = _run_ranks(world)
    for r in range(world):
        np.testing.assert_allclose(out[r], ref, rtol=0, atol=1e-11)


def test_partials_with_another_ranks_weights_do_not():
    """Negative control: a rank multiplying by another rank's W_o columns is caught."""
    ref = _unsharded()
    out = _run_ranks(2, swap=True)
    assert np.abs(out[0] - ref).max() > 1e-2
