"""Pins of the float64 oracle against results fixed by mathematics or by a library routine.

Each test would fail for a plausible slip in the oracle: a wrong scale or sign, a
transposed operand, a wrong GQA head map, a wrong page/slot index, an off-by-one in the
block mask, a dropped term in the split-KV merge.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from ragged_attention_encoder_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _sdpa(q, k, v, mask=None, scale=None):
    """torch's float64 CPU SDPA on one batch: q [n, Hq, d], k/v [L, Hkv, d] -> [n, Hq, d]."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    m = None if mask is None else torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale,
                                       enable_gqa=q.shape[1] != k.shape[1])
    return o[0].permute(1, 0, 2).numpy()


# ----------------------------------------------------------------------------- closed forms

def test_constant_v_returns_v():
    q = RNG.standard_normal((7, 64))
    k = RNG.standard_normal((33, 64))
    c = RNG.standard_normal(64)
    v = np.tile(c, (33, 1))
    out = oracle.attention_rows(q, k, v, 1 / 8.0)
    assert np.allclose(out, c[None, :], atol=1e-13, rtol=0)
    vis = oracle.block_causal_visible(33, 4)[:7]
    out = oracle.attention_rows(q, k, v, 1 / 8.0, vis)
    assert np.allclose(out, c[None, :], atol=1e-13, rtol=0)


def test_single_key_returns_its_value():
    q = RNG.standard_normal((5, 128))
    k = RNG.standard_normal((1, 128))
    v = RNG.standard_normal((1, 128))
    out = oracle.attention_rows(q, k, v, 0.3)
    assert np.allclose(out, np.tile(v, (5, 1)), atol=1e-14, rtol=0)


def test_zero_query_gives_mean_of_visible_values():
    L, bs = 19, 4
    k = RNG.standard_normal((L, 16))
    v = RNG.standard_normal((L, 16))
    q = np.zeros((L, 16))
    out = oracle.attention_rows(q, k, v, 1.0, oracle.block_causal_visible(L, bs))
    for i in range(L):
        last_block_end = min(L, (i // bs + 1) * bs)
        assert np.allclose(out[i], v[:last_block_end].mean(axis=0), atol=1e-13)


def test_two_key_closed_form_golden():
    """A worked example with a result in closed form (softmax of two scores is a sigmoid)."""
    with open(os.path.join(GOLDEN, "two_key_closed_form.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    v = np.array(g["v"], dtype=np.float64)
    out = oracle.attention_rows(q, k, v, g["scale"])
    assert np.allclose(out, np.array(g["expected"]), atol=1e-14, rtol=0)
    # and the same identity on random data: o = sigmoid(s1 - s2) v1 + sigmoid(s2 - s1) v2
    q = RNG.standard_normal((3, 8))
    k = RNG.standard_normal((2, 8))
    v = RNG.standard_normal((2, 8))
    s = q @ k.T * 0.5
    sig = 1.0 / (1.0 + np.exp(-(s[:, 0] - s[:, 1])))
    expect = sig[:, None] * v[0] + (1 - sig)[:, None] * v[1]
    assert np.allclose(oracle.attention_rows(q, k, v, 0.5), expect, atol=1e-14)


def test_no_visible_key_gives_zero_and_empty_query():
    q = RNG.standard_normal((2, 8))
    k = RNG.standard_normal((3, 8))
    v = RNG.standard_normal((3, 8))
    vis = np.zeros((2, 3), dtype=bool)
    assert np.all(oracle.attention_rows(q, k, v, 1.0, vis) == 0)
    assert oracle.attention_rows(q[:0], k, v, 1.0).shape == (0, 8)
    assert np.all(oracle.attention_rows(q, k[:0], v[:0], 1.0) == 0)


# ------------------------------------------------------------------------- library special case

@pytest.mark.parametrize("hq,hkv,d", [(4, 2, 64), (8, 8, 32), (8, 1, 16), (6, 3, 128)])
def test_paged_cross_matches_sdpa(hq, hkv, d):
    case = inputs.paged_case(11 + hq, q_lens=(0, 5, 4), ctx_lens=(1, 40, 4), num_qo_heads=hq,
                             num_kv_heads=hkv, head_dim=d, page_size=16)
    kp = inputs.nan_pool(case.num_pages, hkv, 16, d)
    vp = inputs.nan_pool(case.num_pages, hkv, 16, d)
    kp, vp = oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)
    out = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                       case.kv_page_indices, case.kv_len)
    qf, kf, vf = (oracle.as_f64(t) for t in (case.q, case.k_ctx, case.v_ctx))
    for b in range(case.batch):
        q0, q1 = case.qo_indptr[b], case.qo_indptr[b + 1]
        c0, c1 = case.cu_enc[b], case.cu_enc[b + 1]
        if q1 == q0:
            continue
        ref = _sdpa(qf[q0:q1], kf[c0:c1], vf[c0:c1])
        assert np.allclose(out[q0:q1], ref, atol=1e-12, rtol=1e-12)


@pytest.mark.parametrize("bs", [1, 3, 4, 16, 64])
def test_ragged_block_causal_matches_sdpa(bs):
    case = inputs.ragged_case(5, span_lens=[1, 17, 40, 5], num_qo_heads=4, num_kv_heads=2,
                              head_dim=32, block_size=bs)
    out = oracle.ragged_block_causal_attention(case.q, case.k, case.v, case.cu_q, bs)
    qf, kf, vf = (oracle.as_f64(t) for t in (case.q, case.k, case.v))
    for r in range(case.num_spans):
        a, b = case.cu_q[r], case.cu_q[r + 1]
        L = b - a
        mask = np.zeros((L, L), dtype=bool)
        for i in range(L):              # brute force: enumerate the pairs one by one
            for j in range(L):
                mask[i, j] = (j // bs) <= (i // bs)
        ref = _sdpa(qf[a:b], kf[a:b], vf[a:b], mask)
        assert np.allclose(out[a:b], ref, atol=1e-12, rtol=1e-12)
    rows = [(0, 0), (20, 3), (57, 1), (62, 2)]
    got = oracle.ragged_block_causal_rows(case.q, case.k, case.v, case.cu_q, bs, rows)
    for n, (t, h) in enumerate(rows):
        assert np.allclose(got[n], out[t, h], atol=1e-13, rtol=0)


def test_ragged_cross_matches_sdpa():
    case = inputs.ragged_case(6, span_lens=[3, 1, 9], kv_span_lens=[30, 2, 17], num_qo_heads=8,
                              num_kv_heads=4, head_dim=64, block_size=0)
    out = oracle.ragged_cross_attention(case.q, case.k, case.v, case.cu_q, case.cu_kv)
    qf, kf, vf = (oracle.as_f64(t) for t in (case.q, case.k, case.v))
    for r in range(case.num_spans):
        a, b = case.cu_q[r], case.cu_q[r + 1]
        c, e = case.cu_kv[r], case.cu_kv[r + 1]
        assert np.allclose(out[a:b], _sdpa(qf[a:b], kf[c:e], vf[c:e]), atol=1e-12)


def test_explicit_scale_matches_sdpa():
    q = RNG.standard_normal((4, 2, 16))
    k = RNG.standard_normal((9, 2, 16))
    v = RNG.standard_normal((9, 2, 16))
    for h in range(2):
        got = oracle.attention_rows(q[:, h], k[:, h], v[:, h], 0.71)
        ref = _sdpa(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], scale=0.71)[:, 0]
        assert np.allclose(got, ref, atol=1e-12)


# ------------------------------------------------------------------------------- block mask

@pytest.mark.parametrize("bs", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("L", [1, 2, 5, 8, 13, 20])
def test_block_mask_brute_force(L, bs):
    # Walk the span position by position, opening a new block every bs positions.
    block_of = []
    blk, filled = 0, 0
    for _ in range(L):
        if filled == bs:
            blk, filled = blk + 1, 0
        block_of.append(blk)
        filled += 1
    expect = np.array([[block_of[j] <= block_of[i] for j in range(L)] for i in range(L)])
    assert np.array_equal(oracle.block_causal_visible(L, bs), expect)


def test_block_mask_special_cases():
    for L in (1, 7, 30):
        assert np.array_equal(oracle.block_causal_visible(L, 1), np.tril(np.ones((L, L), bool)))
        assert oracle.block_causal_visible(L, L).all()
        assert oracle.block_causal_visible(L, L + 5).all()
        assert oracle.block_causal_visible(L, 0).all()
    # bs = 1 is the textbook causal mask: compare with SDPA's own causal mode
    q = RNG.standard_normal((12, 1, 8))
    k = RNG.standard_normal((12, 1, 8))
    v = RNG.standard_normal((12, 1, 8))
    got = oracle.ragged_block_causal_attention(q, k, v, [0, 12], 1)
    qt, kt, vt = (torch.from_numpy(x).permute(1, 0, 2)[None] for x in (q, k, v))
    ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)[0].permute(1, 0, 2).numpy()
    assert np.allclose(got, ref, atol=1e-12)


# ----------------------------------------------------------------------------------- paging

def _oracle_pools(case):
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    return oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                case.kv_page_indices, kp, vp)


def test_context_write_places_every_token_and_nothing_else():
    case = inputs.paged_case(21, q_lens=[1, 1, 1], ctx_lens=[7, 16, 33], num_qo_heads=2,
                             num_kv_heads=2, head_dim=8, page_size=16, pool_pages=9)
    kp, vp = _oracle_pools(case)
    touched = np.zeros((case.num_pages, 16), dtype=bool)
    for b in range(case.batch):
        pages = case.kv_page_indices[case.kv_page_indptr[b]:case.kv_page_indptr[b + 1]]
        # walk the request's pages in order; page i holds tokens [16 i, 16 i + 16)
        for i, page in enumerate(pages):
            for slot in range(16):
                tok = 16 * i + slot
                if tok >= case.kv_len[b]:
                    continue
                touched[page, slot] = True
                src = case.cu_enc[b] + tok
                assert torch.equal(kp[page, :, slot].view(torch.int16),
                                   case.k_ctx[src].view(torch.int16))
                assert torch.equal(vp[page, :, slot].view(torch.int16),
                                   case.v_ctx[src].view(torch.int16))
    for pool in (kp, vp):
        bits = pool.view(torch.int16).numpy().transpose(0, 2, 1, 3)   # [page, slot, Hkv, d]
        assert np.all(bits[~touched] == inputs.BF16_NAN_BITS)
    assert touched.sum() == case.kv_len.sum()


def test_gather_reads_back_what_the_context_write_placed():
    """Reading a request's keys through its page list returns, in order, the rows the
    context write (pinned above against a page-walking enumeration) placed: a transposed
    page/slot index or a page list read out of order would return other rows."""
    case = inputs.paged_case(23, q_lens=[1, 1, 1], ctx_lens=[5, 16, 50], num_qo_heads=4,
                             num_kv_heads=2, head_dim=8, page_size=16, pool_pages=10)
    kp, vp = _oracle_pools(case)
    for b in range(case.batch):
        c0, c1 = int(case.cu_enc[b]), int(case.cu_enc[b + 1])
        for pool, src in ((kp, case.k_ctx), (vp, case.v_ctx)):
            got = oracle.gather_paged_kv(pool, case.kv_page_indptr, case.kv_page_indices, b,
                                         int(case.kv_len[b]))
            assert got.shape == (c1 - c0, 2, 8)
            assert np.array_equal(got, src[c0:c1].double().numpy())
    # a prefix of the stream reads the same first rows
    got = oracle.gather_paged_kv(kp, case.kv_page_indptr, case.kv_page_indices, 2, 17)
    assert np.array_equal(got, case.k_ctx[int(case.cu_enc[2]):int(case.cu_enc[2]) + 17]
                          .double().numpy())


def test_page_permutation_invariance():
    case = inputs.paged_case(22, q_lens=[2, 3], ctx_lens=[20, 45], num_qo_heads=4, num_kv_heads=2,
                             head_dim=16, page_size=16, pool_pages=12)
    kp, vp = _oracle_pools(case)
    ref = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                       case.kv_page_indices, case.kv_len)
    perm = np.random.default_rng(3).permutation(case.num_pages)   # new id of page p
    kp2 = torch.empty_like(kp)
    vp2 = torch.empty_like(vp)
    kp2[torch.from_numpy(perm)] = kp
    vp2[torch.from_numpy(perm)] = vp
    idx2 = perm[case.kv_page_indices].astype(np.int32)
    got = oracle.paged_cross_attention(case.q, kp2, vp2, case.qo_indptr, case.kv_page_indptr,
                                       idx2, case.kv_len)
    assert np.array_equal(got, ref)


def test_paged_rows_match_full():
    case = inputs.paged_case(23, q_lens=[3, 2, 4], ctx_lens=[5, 50, 17], num_qo_heads=6,
                             num_kv_heads=3, head_dim=32, page_size=16)
    kp, vp = _oracle_pools(case)
    full = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len)
    rows = [(0, 0), (2, 5), (4, 3), (8, 1)]
    got = oracle.paged_cross_attention_rows(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                            case.kv_page_indices, case.kv_len, rows)
    for n, (t, h) in enumerate(rows):
        assert np.allclose(got[n], full[t, h], atol=1e-13, rtol=0)


def test_empty_query_span_writes_nothing():
    case = inputs.paged_case(24, q_lens=[0, 2, 0], ctx_lens=[3, 4, 5], num_qo_heads=2,
                             num_kv_heads=1, head_dim=8, page_size=16)
    kp, vp = _oracle_pools(case)
    out = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                       case.kv_page_indices, case.kv_len)
    assert out.shape == (2, 2, 8)
    assert np.all(np.isfinite(out))


# -------------------------------------------------------------------------------------- GQA

def test_gqa_equals_repeated_kv_heads():
    case = inputs.ragged_case(7, span_lens=[9, 14], num_qo_heads=8, num_kv_heads=2, head_dim=16,
                              block_size=4)
    out = oracle.ragged_block_causal_attention(case.q, case.k, case.v, case.cu_q, 4)
    k_rep = case.k.repeat_interleave(4, dim=1)
    v_rep = case.v.repeat_interleave(4, dim=1)
    mha = oracle.ragged_block_causal_attention(case.q, k_rep, v_rep, case.cu_q, 4)
    assert np.array_equal(out, mha)
    # and a different head map would give a different answer (the pin has teeth)
    k_tile = case.k.repeat(1, 4, 1)
    v_tile = case.v.repeat(1, 4, 1)
    other = oracle.ragged_block_causal_attention(case.q, k_tile, v_tile, case.cu_q, 4)
    assert not np.allclose(out, other)


# ------------------------------------------------------------------------------ split merge

@pytest.mark.parametrize("cuts", [[], [10], [1, 2, 3], [5, 30, 31, 47]])
def test_merge_of_splits_equals_full_attention(cuts):
    L = 48
    q = RNG.standard_normal((6, 32)) * 3
    k = RNG.standard_normal((L, 32))
    v = RNG.standard_normal((L, 32))
    full = oracle.attention_rows(q, k, v, 0.25)
    edges = [0] + cuts + [L]
    parts, lses = [], []
    for a, b in zip(edges[:-1], edges[1:]):
        o, lse = oracle.partial_attention_with_lse(q, k[a:b], v[a:b], 0.25)
        parts.append(o)
        lses.append(lse)
    merged = oracle.merge_partials(np.stack(parts), np.stack(lses))
    assert np.allclose(merged, full, atol=1e-13)
    # the log-sum-exp itself, against a direct sum
    o, lse = oracle.partial_attention_with_lse(q, k, v, 0.25)
    assert np.allclose(lse, np.log(np.exp(q @ k.T * 0.25).sum(axis=1)), atol=1e-12)


def test_merge_with_empty_split():
    q = RNG.standard_normal((2, 8))
    k = RNG.standard_normal((5, 8))
    v = RNG.standard_normal((5, 8))
    o1, l1 = oracle.partial_attention_with_lse(q, k, v, 1.0)
    o2, l2 = oracle.partial_attention_with_lse(q, k[:0], v[:0], 1.0)
    assert np.all(np.isneginf(l2))
    merged = oracle.merge_partials(np.stack([o2, o1]), np.stack([l2, l1]))
    assert np.allclose(merged, o1, atol=1e-14)
    assert np.all(oracle.merge_partials(np.stack([o2]), np.stack([l2])) == 0)


# ---------------------------------------------------------------------------------- inputs

def test_workload_shapes():
    c1 = inputs.workload(1)
    assert c1.kv_len.tolist() == [7, 13] and c1.num_pages == 8 and c1.total_q == 2
    assert len(set(c1.kv_page_indices.tolist())) == 2
    c2 = inputs.workload(2)
    assert c2.kv_page_indices.shape[0] == 64 * 94 and c2.num_pages == 16384
    assert len(set(c2.kv_page_indices.tolist())) == 64 * 94
    c3 = inputs.workload(3)
    assert c3.batch == 32 and 1 <= c3.qo_indptr[1:].min() and c3.num_kv_heads == 8
    q_len = np.diff(c3.qo_indptr)
    assert q_len.min() >= 1 and q_len.max() <= 128
    assert c3.kv_len.min() >= 256 and c3.kv_len.max() <= 4096


def test_tiny_workload_oracle_golden():
    """Regression pin: the oracle's output on the tiny workload (file written by
    tests/golden/make_golden.py, which calls only the oracle)."""
    with open(os.path.join(GOLDEN, "tiny_paged_decode.json")) as f:
        g = json.load(f)
    case = inputs.workload(1)
    kp, vp = _oracle_pools(case)
    out = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                       case.kv_page_indices, case.kv_len)
    assert np.allclose(out, np.array(g["out"]), atol=1e-12, rtol=0)
    assert math.isclose(float(np.abs(out).sum()), g["abs_sum"], rel_tol=1e-12)


# ---------------------------------------------- paged causal self-attention and the append

def _causal_case(seed, qlens, kvlens, hq=4, hkv=2, d=16, page_size=16, pool_pages=None):
    case = inputs.paged_case(seed, q_lens=qlens, ctx_lens=kvlens, num_qo_heads=hq,
                             num_kv_heads=hkv, head_dim=d, page_size=page_size,
                             pool_pages=pool_pages)
    kp, vp = _oracle_pools(case)
    return case, kp, vp


def _causal(case, kp, vp):
    return oracle.paged_causal_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                         case.kv_page_indices, case.kv_len)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 1)])
def test_paged_causal_prefill_is_sdpa_causal(hq, hkv):
    """A step whose queries are its whole stream (qlen == kv_len) is ordinary causal
    self-attention over the stream, which torch computes with is_causal=True."""
    lens = [1, 9, 33]
    case, kp, vp = _causal_case(40 + hq, lens, lens, hq, hkv)
    out = _causal(case, kp, vp)
    qf, kf, vf = (oracle.as_f64(t) for t in (case.q, case.k_ctx, case.v_ctx))
    for b in range(case.batch):
        q0, q1 = case.qo_indptr[b], case.qo_indptr[b + 1]
        c0, c1 = case.cu_enc[b], case.cu_enc[b + 1]
        qt = torch.from_numpy(qf[q0:q1]).permute(1, 0, 2)[None]
        kt = torch.from_numpy(kf[c0:c1]).permute(1, 0, 2)[None]
        vt = torch.from_numpy(vf[c0:c1]).permute(1, 0, 2)[None]
        ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                             enable_gqa=hq != hkv)[0].permute(1, 0, 2).numpy()
        assert np.allclose(out[q0:q1], ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("qlen,kv_len", [(1, 1), (1, 9), (4, 4), (3, 10), (7, 7), (5, 6)])
def test_causal_append_mask_brute_force(qlen, kv_len):
    """Walk the stream: its last qlen tokens are the queries, each sees every token up to
    and including its own position.  qlen == kv_len is the textbook lower triangle."""
    expect = np.zeros((qlen, kv_len), dtype=bool)
    for i in range(qlen):
        own = kv_len - qlen + i             # stream position of query i
        for j in range(kv_len):
            expect[i, j] = j <= own
    got = oracle.causal_append_visible(qlen, kv_len)
    assert np.array_equal(got, expect)
    if qlen == kv_len:
        assert np.array_equal(got, np.tril(np.ones((qlen, qlen), bool)))
    if qlen == 1:
        assert got.all()


def test_paged_causal_query_sees_the_stream_up_to_itself():
    """Query i of a step is the stream's token kv_len - qlen + i: its result equals
    cross-attention (pinned to SDPA) of that query over the stream cut just after it."""
    case, kp, vp = _causal_case(44, [3, 1, 7, 5], [20, 5, 40, 5])
    out = _causal(case, kp, vp)
    for b in range(case.batch):
        q0, q1 = int(case.qo_indptr[b]), int(case.qo_indptr[b + 1])
        qlen, kvl = q1 - q0, int(case.kv_len[b])
        p0, p1 = int(case.kv_page_indptr[b]), int(case.kv_page_indptr[b + 1])
        for i in range(qlen):
            t = q0 + i
            ref = oracle.paged_cross_attention(case.q[t:t + 1], kp, vp, [0, 1], [0, p1 - p0],
                                               case.kv_page_indices[p0:p1], [kvl - qlen + i + 1])
            assert np.allclose(out[t], ref[0], atol=1e-13, rtol=0)


def test_paged_causal_single_query_steps_are_cross_attention():
    case, kp, vp = _causal_case(45, [1, 1, 1], [7, 16, 50])
    causal = _causal(case, kp, vp)
    cross = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                         case.kv_page_indices, case.kv_len)
    assert np.allclose(causal, cross, atol=1e-13, rtol=0)


def test_paged_causal_rows_match_full():
    case, kp, vp = _causal_case(47, [4, 2, 6], [30, 2, 70], hq=6, hkv=3, d=32)
    full = _causal(case, kp, vp)
    rows = [(0, 0), (3, 5), (4, 2), (5, 1), (11, 4)]
    got = oracle.paged_causal_attention_rows(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                             case.kv_page_indices, case.kv_len, rows)
    for n, (t, h) in enumerate(rows):
        assert np.allclose(got[n], full[t, h], atol=1e-13, rtol=0)


def _split_stream(case, n_new):
    """The first kv_len - n tokens of every request (packed) and the last n (packed)."""
    pre, new, cu_pre, cu_new = [], [], [0], [0]
    for b in range(case.batch):
        c0, c1 = int(case.cu_enc[b]), int(case.cu_enc[b + 1])
        pre.append(torch.arange(c0, c1 - n_new[b]))
        new.append(torch.arange(c1 - n_new[b], c1))
        cu_pre.append(cu_pre[-1] + c1 - n_new[b] - c0)
        cu_new.append(cu_new[-1] + n_new[b])
    return torch.cat(pre), torch.cat(new), np.array(cu_pre), np.array(cu_new)


def test_append_completes_the_context_write_bit_for_bit():
    """Context write of each stream's first tokens, then the append of its last ones, leaves
    exactly the pools of one context write of the whole streams (NaN sentinel elsewhere)."""
    case = inputs.paged_case(46, q_lens=[3, 1, 5, 0], ctx_lens=[20, 1, 37, 16], num_qo_heads=2,
                             num_kv_heads=2, head_dim=8, page_size=16, pool_pages=12)
    full_k, full_v = _oracle_pools(case)
    n_new = [3, 1, 5, 0]
    pre, new, cu_pre, cu_new = _split_stream(case, n_new)
    kp = inputs.nan_pool(case.num_pages, 2, 16, 8)
    vp = inputs.nan_pool(case.num_pages, 2, 16, 8)
    kp, vp = oracle.context_write(case.k_ctx[pre], case.v_ctx[pre], cu_pre, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)
    kp, vp = oracle.append_kv(case.k_ctx[new], case.v_ctx[new], cu_new, case.kv_page_indptr,
                              case.kv_page_indices, case.kv_len, kp, vp)
    assert torch.equal(kp.view(torch.int16), full_k.view(torch.int16))
    assert torch.equal(vp.view(torch.int16), full_v.view(torch.int16))


def test_two_appends_equal_one():
    case = inputs.paged_case(48, q_lens=[1, 1], ctx_lens=[19, 34], num_qo_heads=2,
                             num_kv_heads=1, head_dim=8, page_size=16, pool_pages=6)
    pre, new, cu_pre, cu_new = _split_stream(case, [3, 2])
    kp = inputs.nan_pool(case.num_pages, 1, 16, 8)
    vp = inputs.nan_pool(case.num_pages, 1, 16, 8)
    kp, vp = oracle.context_write(case.k_ctx[pre], case.v_ctx[pre], cu_pre, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)
    once = oracle.append_kv(case.k_ctx[new], case.v_ctx[new], cu_new, case.kv_page_indptr,
                            case.kv_page_indices, case.kv_len, kp, vp)
    # the same tokens in two steps: the first two of each request, then the rest
    kl_mid = case.kv_len - np.array([1, 1])
    first = torch.cat([new[0:2], new[3:4]])
    second = torch.cat([new[2:3], new[4:5]])
    kp2, vp2 = oracle.append_kv(case.k_ctx[first], case.v_ctx[first], [0, 2, 3],
                                case.kv_page_indptr, case.kv_page_indices, kl_mid, kp, vp)
    kp2, vp2 = oracle.append_kv(case.k_ctx[second], case.v_ctx[second], [0, 1, 2],
                                case.kv_page_indptr, case.kv_page_indices, case.kv_len, kp2, vp2)
    assert torch.equal(kp2.view(torch.int16), once[0].view(torch.int16))
    assert torch.equal(vp2.view(torch.int16), once[1].view(torch.int16))


# ----------------------------------------------------------- K/V projection of the context

def _proj_inputs(seed, tokens, hidden, hkv, d, bias=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(tokens, hidden, generator=g).to(torch.bfloat16)
    wk = (torch.randn(hkv * d, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    wv = (torch.randn(hkv * d, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    bk = torch.randn(hkv * d, generator=g).to(torch.bfloat16) if bias else None
    bv = torch.randn(hkv * d, generator=g).to(torch.bfloat16) if bias else None
    return x, wk, bk, wv, bv


def test_projection_of_a_one_hot_row_is_a_weight_column():
    """x = e_i gives k = W_k[:, i] + b_k: fixes which index of W is contracted (W is not
    square here, so a transposed product could not even be formed)."""
    hidden, hkv, d = 96, 2, 16
    _, wk, bk, wv, bv = _proj_inputs(60, 1, hidden, hkv, d)
    x = torch.eye(hidden, dtype=torch.bfloat16)[[0, 7, 95]]
    k, v = oracle.project_kv(x, wk, bk, wv, bv, hkv, d)
    for n, i in enumerate([0, 7, 95]):
        assert np.array_equal(k[n].reshape(-1), oracle.as_f64(wk)[:, i] + oracle.as_f64(bk))
        assert np.array_equal(v[n].reshape(-1), oracle.as_f64(wv)[:, i] + oracle.as_f64(bv))


def test_projection_with_identity_weights_returns_the_rows():
    hkv, d = 4, 16
    x = _proj_inputs(61, 5, hkv * d, hkv, d)[0]
    eye = torch.eye(hkv * d, dtype=torch.bfloat16)
    k, v = oracle.project_kv(x, eye, None, eye, None, hkv, d)
    assert np.array_equal(k, oracle.as_f64(x).reshape(5, hkv, d))
    assert np.array_equal(v, k)


def test_projection_is_affine_and_zero_weights_give_the_bias():
    hidden, hkv, d = 64, 2, 32
    x1, wk, bk, wv, bv = _proj_inputs(62, 6, hidden, hkv, d)
    x2 = _proj_inputs(63, 6, hidden, hkv, d)[0]
    k1, v1 = oracle.project_kv(x1, wk, bk, wv, bv, hkv, d)
    k2, v2 = oracle.project_kv(x2, wk, bk, wv, bv, hkv, d)
    k3, v3 = oracle.project_kv(x1.double() * 3 + x2.double(), wk, bk, wv, bv, hkv, d)
    b = oracle.as_f64(bk).reshape(hkv, d)
    assert np.allclose(k3 - b, 3 * (k1 - b) + (k2 - b), atol=1e-12)
    zero = torch.zeros_like(wk)
    k0, v0 = oracle.project_kv(x1, zero, bk, zero, None, hkv, d)
    assert np.array_equal(k0, np.broadcast_to(b, k0.shape)) and not np.any(v0)


def test_every_exported_oracle_function_has_a_pin_here():
    """Every function the oracle exports is called by at least one test of this file."""
    import inspect
    import re
    src = inspect.getsource(inspect.getmodule(test_every_exported_oracle_function_has_a_pin_here))
    body = src.split("def test_every_exported_oracle_function_has_a_pin_here")[0]
    exported = [n for n, f in vars(oracle).items()
                if callable(f) and not n.startswith("_") and getattr(f, "__module__", "").startswith("oracle")]
    assert exported
    missing = [n for n in exported if not re.search(r"oracle\." + n + r"\(", body)]
    assert not missing, f"oracle functions without a pin: {missing}"
