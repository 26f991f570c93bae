"""Paged causal self-attention and the K/V append on the GPU, against the float64 oracle.

A step's queries are the last tokens of each request's stream (their K/V appended first);
query i sees the stream up to its own token.  Pools start as bf16 NaN so that a stray read
of an untouched slot poisons the output.
"""
import numpy as np
import pytest
import torch

import oracle
from ragged_attention_encoder_b200 import Context, inputs

from gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _stream_case(seed, q_lens, kv_lens, hq, hkv, d, P, pool_pages=None):
    return inputs.paged_case(seed, q_lens=q_lens, ctx_lens=kv_lens, num_qo_heads=hq,
                             num_kv_heads=hkv, head_dim=d, page_size=P, pool_pages=pool_pages)


def _split(case):
    """Packed rows of each stream's first kv_len - qlen tokens and of its last qlen."""
    q_len = np.diff(case.qo_indptr)
    pre, new = [], []
    for b in range(case.batch):
        c0, c1 = int(case.cu_enc[b]), int(case.cu_enc[b + 1])
        pre.append(torch.arange(c0, c1 - int(q_len[b])))
        new.append(torch.arange(c1 - int(q_len[b]), c1))
    pre, new = torch.cat(pre), torch.cat(new)
    cu_pre = np.concatenate([[0], np.cumsum(np.diff(case.cu_enc) - q_len)]).astype(np.int32)
    return pre, new, cu_pre


def _write_then_append(case, ctx):
    """Context write of every stream's prefix, then the append of the step's own tokens."""
    pre, new, cu_pre = _split(case)
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, "cuda")
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, "cuda")
    ctx.write_context(case.k_ctx[pre].cuda(), case.v_ctx[pre].cuda(), cu_pre, case.kv_page_indptr,
                      case.kv_page_indices, kp, vp)
    ctx.append_kv(case.k_ctx[new].cuda(), case.v_ctx[new].cuda(), case.qo_indptr,
                  case.kv_page_indptr, case.kv_page_indices, case.kv_len, kp, vp)
    return kp, vp


def _oracle_pools(case):
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    return oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                case.kv_page_indices, kp, vp)


def _run(case, ctx, kp, vp):
    plan = ctx.plan_paged(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices, case.kv_len,
                          case.num_pages, causal=True)
    q = case.q.cuda()
    out = torch.full_like(q, float("nan"))
    ctx.run_paged(plan, q, kp, vp, out)
    torch.cuda.synchronize()
    ctx.check_device_status()
    return out, plan


def test_append_is_bit_exact():
    case = _stream_case(300, [3, 1, 17, 0, 40], [20, 1, 70, 16, 41], 4, 2, 64, 16)
    ctx = Context(4, 2, 64, 16)
    kp, vp = _write_then_append(case, ctx)
    torch.cuda.synchronize()
    rk, rv = _oracle_pools(case)
    assert torch.equal(kp.cpu().view(torch.int16), rk.view(torch.int16))
    assert torch.equal(vp.cpu().view(torch.int16), rv.view(torch.int16))


def test_append_rejects_more_tokens_than_the_stream():
    case = _stream_case(301, [2], [5], 2, 2, 64, 16)
    ctx = Context(2, 2, 64, 16)
    kp = inputs.nan_pool(case.num_pages, 2, 16, 64, "cuda")
    k_new = torch.zeros(6, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="more tokens"):
        ctx.append_kv(k_new, k_new, [0, 6], case.kv_page_indptr, case.kv_page_indices,
                      case.kv_len, kp, kp.clone())


@pytest.mark.parametrize("hq,hkv,d,P,q_lens,kind", [
    (20, 20, 64, 16, [1] * 6, 1),                 # decode steps: CUDA-core kernel
    (8, 4, 128, 16, [4, 1, 2, 3], 1),             # up to 8 rows per KV head: CUDA-core kernel
    (8, 2, 128, 32, [40, 3, 70], 2),              # chunks: 128-row query tiles
    (32, 8, 128, 16, [128, 5, 64, 100], 2),
    (16, 16, 64, 64, [33, 1, 90], 2),
])
def test_paged_causal_matches_oracle(hq, hkv, d, P, q_lens, kind):
    rng = np.random.default_rng(sum(q_lens) + hq + d)
    kv_lens = [int(q + rng.integers(0, 900)) for q in q_lens]
    case = _stream_case(310 + hq + d + P, q_lens, kv_lens, hq, hkv, d, P)
    ctx = Context(hq, hkv, d, P)
    kp, vp = _write_then_append(case, ctx)
    out, plan = _run(case, ctx, kp, vp)
    assert plan.kernel_kind == kind
    rk, rv = _oracle_pools(case)
    ref = oracle.paged_causal_attention(case.q, rk, rv, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    assert_close(out, ref, what=f"causal {hq}/{hkv} d={d} P={P} q={q_lens}")


@pytest.mark.parametrize("num_sms", [1, 3, 7])
@pytest.mark.parametrize("qmax", [2, 96])
def test_paged_causal_with_forced_splits(num_sms, qmax):
    """Small grids cut units inside their keys: rows whose limit falls before a split's keys
    see nothing in that split, and the merge still gives the oracle's result."""
    rng = np.random.default_rng(320 + num_sms + qmax)
    q_lens = [int(x) for x in rng.integers(1, qmax + 1, 5)]
    kv_lens = [q + int(rng.integers(0, 1500)) for q in q_lens]
    case = _stream_case(320 + num_sms + qmax, q_lens, kv_lens, 8, 2, 128, 16)
    ctx = Context(8, 2, 128, 16, num_sms=num_sms)
    kp, vp = _write_then_append(case, ctx)
    out, plan = _run(case, ctx, kp, vp)
    rk, rv = _oracle_pools(case)
    ref = oracle.paged_causal_attention(case.q, rk, rv, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    assert_close(out, ref, what=f"causal split sms={num_sms} q<={qmax}")


@pytest.mark.parametrize("kv_lens", [[140, 150, 260], [200, 385, 300]])
def test_one_tile_unit_rows_whose_limit_ends_in_the_first_block(kv_lens):
    """One query tile over two or three key blocks, causal: the early queries' limits fall
    before the second block, so every key of that block is masked for those rows."""
    q_lens = [30, 32, 25]
    case = _stream_case(335 + sum(kv_lens), q_lens, kv_lens, 16, 4, 128, 16)
    ctx = Context(16, 4, 128, 16)
    kp, vp = _write_then_append(case, ctx)
    out, plan = _run(case, ctx, kp, vp)
    assert plan.kernel_kind == 2
    rk, rv = _oracle_pools(case)
    ref = oracle.paged_causal_attention(case.q, rk, rv, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    assert_close(out, ref, what=f"causal one tile {kv_lens}")


def test_prefill_whole_stream():
    """qlen == kv_len: the whole stream is new (a prompt's first step)."""
    lens = [1, 128, 300, 77]
    case = _stream_case(330, lens, lens, 16, 4, 128, 16)
    ctx = Context(16, 4, 128, 16)
    kp, vp = _write_then_append(case, ctx)
    out, plan = _run(case, ctx, kp, vp)
    rk, rv = _oracle_pools(case)
    ref = oracle.paged_causal_attention(case.q, rk, rv, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    assert_close(out, ref, what="prefill")


def test_decode_loop_appends_one_token_per_step():
    """Three decode steps: each appends one token per request and attends causally; every
    step matches the oracle on the stream as it stands."""
    full = [40, 1, 17, 300]
    case = _stream_case(340, [1] * 4, full, 8, 8, 64, 16)
    ctx = Context(8, 8, 64, 16)
    steps = 3
    first = [max(n - steps, 0) for n in full]
    cu = case.cu_enc
    kp = inputs.nan_pool(case.num_pages, 8, 16, 64, "cuda")
    vp = inputs.nan_pool(case.num_pages, 8, 16, 64, "cuda")
    pre = torch.cat([torch.arange(int(cu[b]), int(cu[b]) + first[b]) for b in range(4)])
    ctx.write_context(case.k_ctx[pre].cuda(), case.v_ctx[pre].cuda(),
                      np.concatenate([[0], np.cumsum(first)]).astype(np.int32),
                      case.kv_page_indptr, case.kv_page_indices, kp, vp)
    gen = torch.Generator().manual_seed(341)
    for s in range(steps):
        kv_len = np.array([min(first[b] + s + 1, full[b]) for b in range(4)], np.int32)
        grow = np.array([kv_len[b] - min(first[b] + s, full[b]) for b in range(4)], np.int32)
        rows = torch.cat([torch.arange(int(cu[b]) + kv_len[b] - grow[b], int(cu[b]) + kv_len[b])
                          for b in range(4)])
        ap = np.concatenate([[0], np.cumsum(grow)]).astype(np.int32)
        ctx.append_kv(case.k_ctx[rows].cuda(), case.v_ctx[rows].cuda(), ap, case.kv_page_indptr,
                      case.kv_page_indices, kv_len, kp, vp)
        qo = np.arange(5, dtype=np.int32)
        q = torch.randn(4, 8, 64, generator=gen).to(torch.bfloat16)
        plan = ctx.plan_paged(qo, case.kv_page_indptr, case.kv_page_indices, kv_len,
                              case.num_pages, causal=True)
        out = ctx.run_paged(plan, q.cuda(), kp, vp)
        torch.cuda.synchronize()
        ctx.check_device_status()
        rk = inputs.nan_pool(case.num_pages, 8, 16, 64)
        rv = inputs.nan_pool(case.num_pages, 8, 16, 64)
        have = torch.cat([torch.arange(int(cu[b]), int(cu[b]) + kv_len[b]) for b in range(4)])
        rk, rv = oracle.context_write(case.k_ctx[have], case.v_ctx[have],
                                      np.concatenate([[0], np.cumsum(kv_len)]).astype(np.int32),
                                      case.kv_page_indptr, case.kv_page_indices, rk, rv)
        ref = oracle.paged_causal_attention(q, rk, rv, qo, case.kv_page_indptr,
                                            case.kv_page_indices, kv_len)
        assert_close(out, ref, what=f"decode step {s}")


def test_chunked_prefill_workload_sampled():
    """The measured shape: 32 requests append 128-token chunks to streams of 256..4096
    tokens (32/8 heads, d = 128, 16-token pages); sampled rows against the oracle."""
    case = inputs.causal_chunked_prefill()
    ctx = Context(case.num_qo_heads, case.num_kv_heads, case.head_dim, case.page_size)
    kp, vp = _write_then_append(case, ctx)
    out, plan = _run(case, ctx, kp, vp)
    assert plan.kernel_kind == 2
    rk, rv = _oracle_pools(case)
    rng = np.random.default_rng(5)
    rows = [(int(t), int(h)) for t, h in zip(rng.integers(0, case.q.shape[0], 48),
                                            rng.integers(0, case.num_qo_heads, 48))]
    qo = case.qo_indptr
    rows += [(int(qo[b]), 0) for b in range(0, case.batch, 4)]          # first query: shortest prefix
    rows += [(int(qo[b + 1]) - 1, 31) for b in range(0, case.batch, 4)]  # last query: whole stream
    ref = oracle.paged_causal_attention_rows(case.q, rk, rv, qo, case.kv_page_indptr,
                                             case.kv_page_indices, case.kv_len, rows)
    got = torch.stack([out[t, h] for t, h in rows]).float().cpu().numpy()
    assert_close(torch.from_numpy(got), ref, what="chunked prefill rows")
