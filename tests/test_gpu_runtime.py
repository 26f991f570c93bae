"""Runtime behaviour on the GPU: plan slots, staging race, stale plans, status words and the
bounded-wait failure path."""
import numpy as np
import pytest
import torch

from ragged_attention_encoder_b200 import Context, RaeError, _lib, inputs

from gpu_util import assert_close, gpu_pools, oracle_paged

pytestmark = pytest.mark.gpu


def _case(seed, qmax=1):
    return inputs.paged_case(seed, q_lens=(1, qmax, 5), ctx_lens=(20, 400, 5), num_qo_heads=8,
                             num_kv_heads=2, head_dim=64, page_size=16, pool_pages=200)


def test_double_buffered_plans_under_a_busy_stream():
    """plan(N+1) and plan(N+2) are issued while run(N) still waits behind a long kernel on the
    stream; every run must still see its own plan (the staging race of the cross manager)."""
    cases = [_case(200), _case(201, qmax=3), _case(202)]
    span = 130                      # pages reserved per case (5 requests x <= 25 pages)
    num_pages = span * len(cases)
    ctx = Context(8, 2, 64, 16)
    k_pool = inputs.nan_pool(num_pages, 2, 16, 64, "cuda")
    v_pool = inputs.nan_pool(num_pages, 2, 16, 64, "cuda")
    outs = []
    torch.cuda._sleep(200_000_000)   # keep the stream busy for a while
    for i, c in enumerate(cases):
        c.kv_page_indices = np.arange(c.kv_page_indices.size, dtype=np.int32) + span * i
        c.num_pages = num_pages
        ctx.write_context(c.k_ctx.cuda(), c.v_ctx.cuda(), c.cu_enc, c.kv_page_indptr,
                          c.kv_page_indices, k_pool, v_pool)
        plan = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len,
                              num_pages)
        outs.append(ctx.run_paged(plan, c.q.cuda(), k_pool, v_pool))
    torch.cuda.synchronize()
    ctx.check_device_status()
    for c, o in zip(cases, outs):
        assert_close(o, oracle_paged(c), what="double buffer")


def test_stale_plan_is_rejected():
    c = _case(210)
    ctx = Context(8, 2, 64, 16)
    kp, vp = gpu_pools(c, ctx)
    p0 = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages, slot=0)
    ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages, slot=0)
    with pytest.raises(ValueError, match="re-planned"):
        ctx.run_paged(p0, c.q.cuda(), kp, vp)


def test_plan_kind_must_match_run():
    c = _case(211)
    ctx = Context(8, 2, 64, 16)
    kp, vp = gpu_pools(c, ctx)
    rp = ctx.plan_ragged([0, int(c.q.shape[0])], None, 0)   # same query rows: only the kind differs
    with pytest.raises(ValueError, match="kind"):
        ctx.run_paged(rp, c.q.cuda(), kp, vp)


def test_bad_tensors_are_rejected_before_launch():
    c = _case(212)
    ctx = Context(8, 2, 64, 16)
    kp, vp = gpu_pools(c, ctx)
    plan = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages)
    with pytest.raises(ValueError):
        ctx.run_paged(plan, c.q.cuda().float(), kp, vp)
    with pytest.raises(ValueError):
        ctx.run_paged(plan, c.q, kp, vp)          # host tensor
    with pytest.raises(ValueError, match="UNSUPPORTED"):
        Context(8, 3, 64, 16)


def test_buffers_smaller_than_the_plan_are_rejected_before_launch():
    """The pools must hold every page the plan lists, k / v every key its spans read, and q /
    out exactly the plan's query rows; nothing is launched otherwise."""
    c = _case(214)
    ctx = Context(8, 2, 64, 16)
    kp, vp = gpu_pools(c, ctx)
    plan = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages)
    extent = int(np.max(c.kv_page_indices)) + 1
    assert plan.raw.kv_extent == extent
    with pytest.raises(ValueError, match="pools hold"):
        ctx.run_paged(plan, c.q.cuda(), kp[:extent - 1].contiguous(), vp[:extent - 1].contiguous())
    with pytest.raises(ValueError, match="shape"):
        ctx.run_paged(plan, c.q.cuda()[1:].contiguous(), kp, vp)
    with pytest.raises(ValueError, match="shape"):
        ctx.run_paged(plan, c.q.cuda(), kp, vp, torch.empty_like(c.q.cuda())[:, :1].contiguous())
    with pytest.raises(ValueError, match="shape"):
        ctx.run_paged(plan, c.q.cuda(), kp, vp[:, :1].contiguous())
    rp = ctx.plan_ragged([0, 40, 100], [0, 30, 70], 0)
    assert rp.raw.kv_extent == 70
    q = torch.zeros(100, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(69, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="key tokens"):
        ctx.run_ragged(rp, q, k, k.clone())
    torch.cuda.synchronize()
    ctx.check_device_status()


def test_status_word_is_clear_after_normal_runs():
    c = _case(213, qmax=20)
    ctx = Context(8, 2, 64, 16)
    kp, vp = gpu_pools(c, ctx)
    plan = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages)
    for _ in range(3):
        ctx.run_paged(plan, c.q.cuda(), kp, vp)
    ctx.check_device_status()
    assert int(ctx.workspace[:4].view(torch.int32).item()) == 0


def test_bounded_wait_runs_out_and_the_context_recovers():
    """One CTA's producer arms nothing (test build hook): its consumers' waits run out after the
    wait timeout, the kernel exits, the host reads RAE_ERR_DEVICE_TIMEOUT, and the same plan
    then runs exactly (status word and split arrival counters were cleared)."""
    lib = _lib.load_test()
    c = _case(220)
    ctx = Context(8, 2, 64, 16, num_sms=2, library=lib)
    kp, vp = gpu_pools(c, ctx)
    plan = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages)
    assert plan.kernel_kind == 1 and plan.num_ctas == 4 and plan.num_merge_rows > 0
    ref = oracle_paged(c)
    q = c.q.cuda()
    ctx.set_wait_timeout_ns(5_000_000)
    assert lib.rae_test_silence_producer(1) == _lib.RAE_OK
    try:
        ctx.run_paged(plan, q, kp, vp)
        with pytest.raises(RaeError) as info:
            ctx.check_device_status()
        assert info.value.status == _lib.RAE_ERR_DEVICE_TIMEOUT
        assert "site 102" in str(info.value)     # a consumer's wait for a stage to fill
    finally:
        assert lib.rae_test_silence_producer(-1) == _lib.RAE_OK
    ctx.set_wait_timeout_ns(4_000_000_000)
    assert int(ctx.workspace[:4].view(torch.int32).item()) == 0
    for _ in range(2):
        out = ctx.run_paged(plan, q, kp, vp)
        ctx.check_device_status()
        assert_close(out, ref, what="after a timed-out run")


@pytest.mark.parametrize("qmax", [1, 40])
def test_planned_run_calls_replay_from_a_cuda_graph(qmax):
    """Once planned, a run call is a stream-ordered launch and nothing else: a CUDA graph that
    captures several layer calls (decode kernel for one-token queries, the tensor-core kernel
    for packs of up to 40) replays them with outputs bit-identical to eager calls."""
    c = _case(230 + qmax, qmax=qmax)
    ctx = Context(8, 2, 64, 16)
    kp, vp = gpu_pools(c, ctx)
    plan = ctx.plan_paged(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages)
    assert plan.kernel_kind == (1 if qmax == 1 else 2)
    gen = torch.Generator(device="cuda").manual_seed(qmax)
    layers = 4
    qs = [c.q.cuda()] + [torch.randn(c.q.shape, generator=gen, device="cuda").to(torch.bfloat16)
                         for _ in range(layers - 1)]
    eager = [ctx.run_paged(plan, q, kp, vp) for q in qs]
    outs = [torch.empty_like(q) for q in qs]
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for q, o in zip(qs, outs):
            ctx.run_paged(plan, q, kp, vp, o)
    for o in outs:
        o.zero_()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    ctx.check_device_status()
    for e, o in zip(eager, outs):
        assert torch.equal(e, o)
    assert_close(outs[0], oracle_paged(c), what="graph replay")
