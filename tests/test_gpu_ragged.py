"""Cacheless ragged attention on the GPU (block-causal self and two-span cross) vs the oracle."""
import numpy as np
import pytest
import torch

import oracle
from ragged_attention_encoder_b200 import inputs

from gpu_util import assert_close, oracle_ragged, run_ragged

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs", [0, 1, 7, 64, 128, 256, 1000])
def test_block_causal_small_spans(bs):
    case = inputs.ragged_case(100 + bs, span_lens=[1, 2, 127, 128, 129, 300, 513], num_qo_heads=4,
                              num_kv_heads=2, head_dim=64, block_size=bs)
    out, *_ = run_ragged(case)
    assert_close(out, oracle_ragged(case), what=f"bs={bs}")


@pytest.mark.parametrize("hq,hkv,d", [(16, 16, 128), (8, 2, 128), (6, 3, 64), (4, 1, 64)])
def test_block_causal_heads(hq, hkv, d):
    case = inputs.ragged_case(110 + hq + d, span_range=(1, 700), min_total=1500, num_qo_heads=hq,
                              num_kv_heads=hkv, head_dim=d, block_size=256)
    out, *_ = run_ragged(case)
    assert_close(out, oracle_ragged(case), what=f"{hq}/{hkv} d={d}")


def test_ragged_block_causal_workload_sampled():
    """The full packed encoder workload (~64k tokens, block 256) in the benchmark's launch
    configuration; sampled (token, head) rows, including span starts and ends, against the
    oracle computed row by row."""
    case = inputs.workload(4)
    out, plan, *_ = run_ragged(case)
    o = out.float().cpu().numpy()
    assert np.all(np.isfinite(o))
    rng = np.random.default_rng(4)
    rows = []
    for s in rng.choice(case.num_spans, 6, replace=False):
        a, b = int(case.cu_q[s]), int(case.cu_q[s + 1])
        for t in (a, a + 1, a + 255, a + 256, (a + b) // 2, b - 1):
            if a <= t < b:
                rows.append((t, int(rng.integers(case.num_qo_heads))))
    ref = oracle.ragged_block_causal_rows(case.q, case.k, case.v, case.cu_q, case.block_size, rows)
    got = np.stack([o[t, h] for t, h in rows])
    assert_close(got, ref, what="workload 4")


@pytest.mark.slow
def test_ragged_block_causal_workload_full():
    """The whole packed encoder workload (31 spans, 65 959 tokens, 16 heads, block 256) in the
    benchmark's launch configuration, compared element by element with the float64 oracle
    (about a minute of host time)."""
    case = inputs.workload(4)
    out, plan, *_ = run_ragged(case)
    assert plan.num_ctas == 148
    assert_close(out, oracle_ragged(case), what="workload 4 (full)")


def test_two_span_cross_tiny():
    case = inputs.ragged_case(120, span_lens=[3, 1, 9, 0, 130, 5, 2, 40],
                              kv_span_lens=[30, 2, 17, 5, 1, 0, 300, 129], num_qo_heads=8,
                              num_kv_heads=4, head_dim=64, block_size=0)
    out, *_ = run_ragged(case)
    assert_close(out, oracle_ragged(case), what="cross tiny")


def test_two_span_cross_multitoken_shapes():
    """Two-span cross-attention with the packed multi-token shapes and contiguous K/V."""
    pc = inputs.workload(3)
    case = inputs.RaggedCase(name="cross", num_qo_heads=pc.num_qo_heads,
                             num_kv_heads=pc.num_kv_heads, head_dim=pc.head_dim, block_size=0,
                             cu_q=pc.qo_indptr, cu_kv=pc.cu_enc, q=pc.q, k=pc.k_ctx, v=pc.v_ctx,
                             self_attention=False)
    out, *_ = run_ragged(case)
    assert_close(out, oracle_ragged(case), what="cross multitoken")


@pytest.mark.parametrize("bs,sms", [(256, 8), (256, 12), (0, 5), (0, 12)])
def test_forced_splits_ragged(bs, sms):
    """A grid with more CTAs than whole units balance over cuts some units' keys: split
    tiles plus the merge."""
    case = inputs.ragged_case(130, span_lens=[1500, 700], num_qo_heads=1, num_kv_heads=1,
                              head_dim=128, block_size=bs)
    out, plan, *_ = run_ragged(case, num_sms=sms)
    assert plan.num_merge_rows > 0
    assert_close(out, oracle_ragged(case), what="ragged split")


def test_ragged_repeat_bit_identical_and_constant_v():
    case = inputs.ragged_case(140, span_lens=[200, 900], num_qo_heads=8, num_kv_heads=8,
                              head_dim=128, block_size=256)
    out1, plan, ctx = run_ragged(case)
    out2 = ctx.run_ragged(plan, case.q.cuda(), case.k.cuda(), case.v.cuda())
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    c = torch.randn(case.head_dim).to(torch.bfloat16)
    case.v = c.expand_as(case.v).contiguous()
    out3, *_ = run_ragged(case)
    o = out3.float().cpu()
    ref = c.float().expand_as(o)
    assert torch.all((o - ref).abs() <= 2.0 ** -7 * ref.abs()), float((o - ref).abs().max())
