"""Paged cross-attention and the context write on the GPU, against the float64 oracle.

Inputs are the seeded workloads of ragged_attention_encoder_b200.inputs; the pools start as
bf16 NaN so that a stray read of an untouched slot poisons the output.
"""
import numpy as np
import pytest
import torch

import oracle
from ragged_attention_encoder_b200 import Context, inputs

from gpu_util import (assert_close, context_for, gpu_pools, oracle_paged, oracle_pools,
                      run_paged)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------- context write

@pytest.mark.parametrize("wl", [1, 3])
def test_context_write_is_bit_exact(wl):
    case = inputs.workload(wl)
    ctx = context_for(case)
    kp, vp = gpu_pools(case, ctx)
    torch.cuda.synchronize()
    rk, rv = oracle_pools(case)
    assert torch.equal(kp.cpu().view(torch.int16), rk.view(torch.int16))
    assert torch.equal(vp.cpu().view(torch.int16), rv.view(torch.int16))


def test_context_write_whisper_pool_is_bit_exact():
    """The full 16384-page pool of the Whisper-large decode workload."""
    case = inputs.workload(2)
    ctx = context_for(case)
    kp, vp = gpu_pools(case, ctx)
    torch.cuda.synchronize()
    rk, rv = oracle_pools(case)
    assert torch.equal(kp.cpu().view(torch.int16), rk.view(torch.int16))
    assert torch.equal(vp.cpu().view(torch.int16), rv.view(torch.int16))


def test_context_write_rejects_duplicate_pages():
    case = inputs.paged_case(31, q_lens=[1, 1], ctx_lens=[10, 10], num_qo_heads=2, num_kv_heads=1,
                             head_dim=64, page_size=16, pool_pages=4)
    ctx = context_for(case)
    kp = inputs.nan_pool(4, 1, 16, 64, "cuda")
    vp = inputs.nan_pool(4, 1, 16, 64, "cuda")
    with pytest.raises(ValueError, match="twice"):
        ctx.write_context(case.k_ctx.cuda(), case.v_ctx.cuda(), case.cu_enc, [0, 1, 2], [3, 3],
                          kp, vp)
    with pytest.raises(ValueError, match="range"):
        ctx.write_context(case.k_ctx.cuda(), case.v_ctx.cuda(), case.cu_enc, [0, 1, 2], [3, 4],
                          kp, vp)
    torch.cuda.synchronize()
    assert torch.all(kp.view(torch.int16) == inputs.BF16_NAN_BITS)


# --------------------------------------------------------------------------- workloads

def test_tiny_paged_decode():
    case = inputs.workload(1)
    out, plan, *_ = run_paged(case)
    assert_close(out, oracle_paged(case), what="tiny")


def test_whisper_large_decode():
    case = inputs.workload(2)
    out, plan, *_ = run_paged(case)
    assert plan.num_merge_rows > 0      # the balanced schedule splits some requests
    assert_close(out, oracle_paged(case), what="whisper")


def test_packed_multitoken_cross():
    case = inputs.workload(3)
    out, plan, *_ = run_paged(case)
    assert_close(out, oracle_paged(case), what="multitoken")


def test_long_context_splitkv_sampled():
    """Full-size long-context workload in the benchmark's launch configuration; sampled rows
    are checked one by one against attention over each request's packed context K/V."""
    case = inputs.workload(5)
    out, plan, *_ = run_paged(case)
    assert plan.num_merge_rows > 0
    g = case.num_qo_heads // case.num_kv_heads
    rng = np.random.default_rng(5)
    o = out.float().cpu().numpy()
    assert np.all(np.isfinite(o))
    scale = 1.0 / np.sqrt(case.head_dim)
    for b in rng.choice(case.batch, 3, replace=False):
        c0, c1 = case.cu_enc[b], case.cu_enc[b + 1]
        for kvh in rng.choice(case.num_kv_heads, 2, replace=False):
            kb = oracle.as_f64(case.k_ctx[c0:c1, kvh])
            vb = oracle.as_f64(case.v_ctx[c0:c1, kvh])
            for t in range(case.qo_indptr[b], case.qo_indptr[b + 1]):
                heads = list(range(kvh * g, kvh * g + g))
                qrows = oracle.as_f64(case.q[t, heads])
                ref = oracle.attention_rows(qrows, kb, vb, scale)
                assert_close(o[t, heads], ref, what=f"req {b} tok {t}")


@pytest.mark.slow
def test_long_context_splitkv_full():
    """The whole long-context workload (8 requests x 4 tokens x 64 heads over 32k-131k keys),
    compared element by element: every (request, KV head) with the float64 oracle's attention
    over the request's context rows (the context write that placed them is bit-exact)."""
    case = inputs.workload(5)
    out, plan, *_ = run_paged(case)
    assert plan.num_merge_rows > 0
    g = case.num_qo_heads // case.num_kv_heads
    ref = np.zeros(tuple(case.q.shape), dtype=np.float64)
    scale = 1.0 / np.sqrt(case.head_dim)
    for b in range(case.batch):
        c0, c1 = int(case.cu_enc[b]), int(case.cu_enc[b + 1])
        t0, t1 = int(case.qo_indptr[b]), int(case.qo_indptr[b + 1])
        for kvh in range(case.num_kv_heads):
            kb = oracle.as_f64(case.k_ctx[c0:c1, kvh])
            vb = oracle.as_f64(case.v_ctx[c0:c1, kvh])
            for h in range(kvh * g, kvh * g + g):
                ref[t0:t1, h] = oracle.attention_rows(oracle.as_f64(case.q[t0:t1, h]), kb, vb,
                                                      scale)
    assert_close(out, ref, what="workload 5 (full)")


# ---------------------------------------------------------------------------- edge cases

@pytest.mark.parametrize("P", [16, 32, 64])
@pytest.mark.parametrize("d", [64, 128])
def test_kv_len_around_page_boundaries(P, d):
    lens = [1, P - 1, P, P + 1, 2 * P + 3]
    case = inputs.paged_case(40 + P + d, q_lens=[1, 2, 1, 3, 1], ctx_lens=lens, num_qo_heads=4,
                             num_kv_heads=2, head_dim=d, page_size=P, pool_pages=64)
    out, *_ = run_paged(case)
    assert_close(out, oracle_paged(case), what=f"P={P} d={d}")


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (8, 2), (8, 1), (6, 2), (40, 5)])
@pytest.mark.parametrize("qmax", [1, 40])
def test_gqa_groups_and_query_lengths(hq, hkv, qmax):
    case = inputs.paged_case(50 + hq + hkv + qmax, q_lens=(0, qmax, 6), ctx_lens=(1, 600, 6),
                             num_qo_heads=hq, num_kv_heads=hkv, head_dim=64, page_size=16)
    out, plan, *_ = run_paged(case)
    assert_close(out, oracle_paged(case), what=f"{hq}/{hkv} q<={qmax}")


@pytest.mark.parametrize("hq,hkv,qlens", [(64, 8, [4, 4, 1, 3]), (64, 8, [8, 5, 2]),
                                          (32, 8, [16, 3, 9]), (32, 2, [2, 1, 4]),
                                          (16, 16, [40, 9, 30]), (16, 1, [1, 1, 2]),
                                          (64, 4, [1, 4, 2])])
@pytest.mark.parametrize("P", [16, 64])
def test_swapped_kernel_for_few_rows(hq, hkv, qlens, P):
    """9..64 query rows per (request, KV head) at d=128 run with keys on the MMA's M side."""
    case = inputs.paged_case(170 + hq + hkv + P + sum(qlens), q_lens=qlens,
                             ctx_lens=(1, 3000, len(qlens)), num_qo_heads=hq, num_kv_heads=hkv,
                             head_dim=128, page_size=P)
    out, plan, *_ = run_paged(case)
    assert plan.kernel_kind == 4
    assert_close(out, oracle_paged(case), what=f"swap {hq}/{hkv} P={P}")


@pytest.mark.parametrize("num_sms", [1, 3, 7])
def test_swapped_kernel_with_forced_splits(num_sms):
    case = inputs.paged_case(180 + num_sms, q_lens=[4, 4, 4], ctx_lens=(2000, 9000, 3),
                             num_qo_heads=64, num_kv_heads=8, head_dim=128, page_size=64)
    out, plan, *_ = run_paged(case, num_sms=num_sms)
    assert plan.kernel_kind == 4
    if num_sms == 7:
        assert plan.num_merge_rows > 0     # this grid cuts units inside their keys
    assert_close(out, oracle_paged(case), what=f"swap split {num_sms}")


@pytest.mark.parametrize("hq,hkv,d,qlens,kind", [
    (8, 1, 128, [1, 1], 1),    # 8 rows per (request, KV head): CUDA-core decode kernel
    (8, 1, 128, [2, 1], 4),    # 16 rows: keys on the MMA M side, 32 columns
    (8, 1, 128, [8, 3], 4),    # 64 rows: keys on the MMA M side, 64 columns
    (8, 1, 128, [9, 2], 2),    # 72 rows: 128-row query tiles
    (8, 1, 64, [2, 1], 2),     # d = 64: no swapped kernel, 128-row query tiles
])
def test_kernel_choice_at_row_boundaries(hq, hkv, d, qlens, kind):
    case = inputs.paged_case(190 + sum(qlens) + d, q_lens=qlens, ctx_lens=(300, 2500, len(qlens)),
                             num_qo_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=16)
    out, plan, *_ = run_paged(case)
    assert plan.kernel_kind == kind
    assert_close(out, oracle_paged(case), what=f"rows boundary {qlens} d={d}")


@pytest.mark.parametrize("qlens,hq,hkv,d,kind", [([0, 1, 0, 1, 0], 20, 20, 64, 1),
                                                 ([0, 4, 0, 2], 64, 8, 128, 4),
                                                 ([0, 37, 0, 5, 0], 32, 8, 128, 2)])
def test_requests_without_queries_between_others(qlens, hq, hkv, d, kind):
    """Requests with no query tokens (their context still in the pool) write nothing and do
    not disturb their neighbours, in every kernel family."""
    case = inputs.paged_case(200 + sum(qlens), q_lens=qlens, ctx_lens=(100, 2000, len(qlens)),
                             num_qo_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=16)
    out, plan, *_ = run_paged(case)
    assert plan.kernel_kind == kind
    assert out.shape[0] == sum(qlens)
    assert_close(out, oracle_paged(case), what=f"empty queries {qlens}")


def test_empty_context_gives_zero():
    case = inputs.paged_case(61, q_lens=[2, 1, 3], ctx_lens=[0, 5, 0], num_qo_heads=4,
                             num_kv_heads=2, head_dim=64, page_size=16, pool_pages=4)
    out, *_ = run_paged(case)
    ref = oracle_paged(case)
    assert np.all(ref[0:2] == 0) and np.all(ref[3:] == 0)
    assert_close(out, ref, what="empty ctx")
    case = inputs.paged_case(62, q_lens=[40, 0, 30], ctx_lens=[0, 5, 700], num_qo_heads=8,
                             num_kv_heads=2, head_dim=128, page_size=16)
    out, plan, *_ = run_paged(case)
    assert plan.kernel_kind == 2
    assert_close(out, oracle_paged(case), what="empty ctx tc")


@pytest.mark.parametrize("ctx_lens,split_sms", [([129, 256], 7), ([257, 300, 383], 11),
                                                ([129, 1000, 513, 640, 900], 20)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("split", [False, True])
def test_one_tile_units_over_several_key_blocks(ctx_lens, split_sms, d, split):
    """Units with one 128-row query tile over two to eight key blocks: even and odd block
    counts, a partial last block, pools of NaN around the pages, with and without cuts inside
    the keys."""
    q_lens = [17 + 5 * i for i in range(len(ctx_lens))]      # 68..148 rows at GQA 4
    case = inputs.paged_case(700 + d + len(ctx_lens), q_lens=q_lens, ctx_lens=ctx_lens,
                             num_qo_heads=16, num_kv_heads=4, head_dim=d, page_size=16)
    cap = {"num_sms": split_sms} if split else {}
    out, plan, *_ = run_paged(case, **cap)
    assert plan.kernel_kind == 2
    if split:
        assert plan.num_merge_rows > 0    # this grid cuts units inside their keys
    assert_close(out, oracle_paged(case), what=f"paired {ctx_lens} d={d} split={split}")


@pytest.mark.parametrize("num_sms,qmax", [(2, 1), (3, 1), (5, 1), (6, 50), (8, 50), (16, 50)])
def test_forced_splits_agree_with_oracle_and_unsplit(num_sms, qmax):
    case = inputs.paged_case(70 + num_sms + qmax, q_lens=(1, qmax, 3), ctx_lens=(300, 3000, 3),
                             num_qo_heads=8, num_kv_heads=2, head_dim=128, page_size=32)
    ref = oracle_paged(case)
    out_split, plan, *_ = run_paged(case, num_sms=num_sms)
    assert plan.num_merge_rows > 0         # a small grid cuts units inside their keys
    assert_close(out_split, ref, what="split")
    out_full, plan_full, *_ = run_paged(case)
    assert_close(out_full, ref, what="unsplit")


@pytest.mark.parametrize("num_sms,split", [(5, False), (148, True)])
def test_output_aligned_to_16_bytes_only(num_sms, split):
    """An output whose address is 16- but not 32-byte aligned takes the kernels' 16-byte store
    path (32-byte stores need 32-byte alignment) and gives the same result, with and without
    split partials."""
    case = inputs.paged_case(91, q_lens=[20, 33, 7], ctx_lens=[300, 1000, 129], num_qo_heads=16,
                             num_kv_heads=4, head_dim=128, page_size=16)
    ctx = context_for(case, num_sms=num_sms)
    kp, vp = gpu_pools(case, ctx)
    plan = ctx.plan_paged(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices, case.kv_len,
                          case.num_pages)
    assert plan.kernel_kind == 2
    assert (plan.num_merge_rows > 0) == split
    q = case.q.cuda()
    buf = torch.full((q.numel() + 16,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[8:8 + q.numel()].view_as(q)
    assert out.data_ptr() % 32 == 16
    ctx.run_paged(plan, q, kp, vp, out)
    torch.cuda.synchronize()
    ctx.check_device_status()
    assert_close(out, oracle_paged(case), what=f"16-byte aligned out, sms={num_sms}")
    aligned, *_ = run_paged(case, num_sms=num_sms)
    assert torch.equal(out.view(torch.int16), aligned.view(torch.int16))


def test_explicit_scale():
    case = inputs.paged_case(81, q_lens=[3, 20], ctx_lens=[100, 257], num_qo_heads=8,
                             num_kv_heads=2, head_dim=64, page_size=16)
    out, *_ = run_paged(case, sm_scale=0.05)
    assert_close(out, oracle_paged(case, scale=0.05), what="scale")


# --------------------------------------------------------------------------- metamorphic

@pytest.mark.parametrize("qmax", [1, 60])
def test_page_permutation_gives_bit_identical_output(qmax):
    case = inputs.paged_case(90 + qmax, q_lens=(1, qmax, 4), ctx_lens=(100, 900, 4),
                             num_qo_heads=8, num_kv_heads=4, head_dim=64, page_size=16)
    out1, *_ = run_paged(case)
    perm = np.random.default_rng(1).permutation(case.num_pages).astype(np.int32)
    case.kv_page_indices = perm[case.kv_page_indices]
    out2, *_ = run_paged(case)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("wl", [2, 3])
def test_repeated_runs_are_bit_identical(wl):
    case = inputs.workload(wl)
    out1, plan, ctx, kp, vp = run_paged(case)
    q = case.q.cuda()
    out2 = ctx.run_paged(plan, q, kp, vp)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_mha_duplicate_of_gqa_matches_oracle():
    case = inputs.paged_case(95, q_lens=(1, 30, 3), ctx_lens=(50, 500, 3), num_qo_heads=8,
                             num_kv_heads=2, head_dim=64, page_size=16)
    ref = oracle_paged(case)
    case.k_ctx = case.k_ctx.repeat_interleave(4, dim=1).contiguous()
    case.v_ctx = case.v_ctx.repeat_interleave(4, dim=1).contiguous()
    case.num_kv_heads = 8
    out, *_ = run_paged(case)
    assert_close(out, ref, what="mha")


def test_constant_v_returns_v():
    case = inputs.paged_case(96, q_lens=(1, 50, 4), ctx_lens=(10, 800, 4), num_qo_heads=8,
                             num_kv_heads=2, head_dim=128, page_size=16)
    c = torch.randn(case.head_dim).to(torch.bfloat16)
    case.v_ctx = c.expand_as(case.v_ctx).contiguous()
    out, *_ = run_paged(case)
    o = out.float().cpu()
    ref = c.float().expand_as(o)
    # P is rounded to bf16 for the tensor core while the row sum adds fp32 values: the
    # result is V up to the bf16 rounding of the probabilities and of the output.
    assert torch.all((o - ref).abs() <= 2.0 ** -7 * ref.abs()), float((o - ref).abs().max())
