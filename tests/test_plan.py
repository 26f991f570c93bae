"""Host-side tests of the C-ABI library: symbol exports and the plan builder (no GPU).

The plan must cover every visible (query token, query head, key) triple exactly once, keep
its split bookkeeping consistent, reject malformed inputs, and be deterministic.
"""
import re
import os

import numpy as np
import pytest

from ragged_attention_encoder_b200 import _lib, build, inputs, plan_paged_host, plan_ragged_host

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session", autouse=True)
def built_library():
    build.build()
    return _lib.load()


def test_library_exports_every_declared_symbol(built_library):
    with open(os.path.join(ROOT, "include", "rae.h")) as f:
        header = f.read()
    declared = set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(rae_\w+)\s*\(", header, flags=re.M))
    assert len(declared) >= 15
    assert declared == set(_lib.SIGNATURES), declared ^ set(_lib.SIGNATURES)
    for name in declared:
        assert hasattr(built_library, name), name


def test_test_build_exports_its_hooks_and_the_product_does_not(built_library):
    with open(os.path.join(ROOT, "include", "rae_test_hooks.h")) as f:
        header = f.read()
    declared = set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(rae_\w+)\s*\(", header, flags=re.M))
    assert declared == set(_lib.TEST_SIGNATURES), declared
    test_lib = _lib.load_test()
    for name in list(_lib.SIGNATURES) + list(declared):
        assert hasattr(test_lib, name), name
    for name in declared:
        assert not hasattr(built_library, name), name


def _tiles_rows(tiles, g):
    """Expand tiles into (token, head, kv0, kv1, tile index).  A tile's unit holds the KV
    heads kvh ... kvh + nkvh - 1 (word 10); its rows are (token, query head), token-major."""
    out = []
    for i, t in enumerate(tiles):
        req, kvh, q0, qn, kv0, kv1, part, split = (int(x) for x in t[:8])
        nkvh = int(t[10])
        assert nkvh >= 1
        hpt = g * nkvh
        for r in range(qn * hpt):
            out.append((q0 + r // hpt, kvh * g + r % hpt, kv0, kv1, i))
    return out


def _check_cta_ptr(p):
    cp = p["cta_ptr"]
    raw = p["raw"]
    assert cp[0] == 0 and cp[-1] == raw.num_tiles
    assert np.all(np.diff(cp) >= 0)
    if raw.num_tiles:
        assert np.all(np.diff(cp) >= 1), "a launched CTA has no tile"


def _check_merge(p, g, hq):
    """Splits of a unit tile its keys in order, share one arrival counter, count themselves,
    and own disjoint partial rows; unsplit units write straight to the output."""
    tiles = p["tiles"]
    units = {}
    for t in tiles:
        req, kvh, q0, qn, kv0, kv1, part, split, munit, nsplit, nkvh = (int(x) for x in t[:11])
        units.setdefault((req, kvh, q0), []).append((split, kv0, kv1, part, qn * nkvh, munit,
                                                     nsplit))
    merge_rows = 0
    seen_parts, seen_units = set(), set()
    for key, pieces in units.items():
        pieces.sort()
        assert [s for s, *_ in pieces] == list(range(len(pieces)))
        for a, b in zip(pieces[:-1], pieces[1:]):
            assert a[2] == b[1], "splits of a unit must be contiguous in keys"
        qn = pieces[0][4]
        if len(pieces) == 1:
            assert pieces[0][3] == -1 and pieces[0][5] == -1 and pieces[0][6] == 1
            continue
        rows = qn * g
        merge_rows += rows
        munits = {pc[5] for pc in pieces}
        assert len(munits) == 1 and min(munits) >= 0
        assert not (munits & seen_units), "two units share an arrival counter"
        seen_units |= munits
        base = pieces[0][3]
        for s, kv0, kv1, part, _, munit, nsplit in pieces:
            assert nsplit == len(pieces)
            assert part == base + s * rows
            for r in range(rows):
                assert part + r not in seen_parts
                seen_parts.add(part + r)
    assert merge_rows == p["raw"].num_merge_rows == p["header"][4]
    assert len(seen_units) == p["header"][10]
    assert seen_units == set(range(len(seen_units)))


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("hq,hkv,d,P", [(4, 2, 64, 16), (8, 1, 128, 32), (6, 6, 64, 64),
                                        (32, 8, 128, 16), (64, 8, 128, 64)])
def test_paged_plan_covers_each_pair_once(seed, hq, hkv, d, P):
    rng = np.random.default_rng(seed * 100 + hq)
    B = int(rng.integers(1, 7))
    q_len = rng.integers(0, 40 if seed % 2 else 3, B)
    kv_len = rng.integers(0, 700, B)
    pages_per = (kv_len + P - 1) // P + rng.integers(0, 2, B)
    indptr = np.concatenate([[0], np.cumsum(pages_per)]).astype(np.int32)
    num_pages = int(indptr[-1]) + 5
    indices = rng.permutation(num_pages)[: indptr[-1]].astype(np.int32)
    qo = np.concatenate([[0], np.cumsum(q_len)]).astype(np.int32)
    # a small grid forces splits even on these small inputs
    p = plan_paged_host(qo, indptr, indices, kv_len, num_pages, num_qo_heads=hq, num_kv_heads=hkv,
                        head_dim=d, page_size=P, num_sms=int(rng.integers(1, 9)))
    g = hq // hkv
    _check_cta_ptr(p)
    cover = {}
    for tok, head, kv0, kv1, i in _tiles_rows(p["tiles"], g):
        cover.setdefault((tok, head), []).append((kv0, kv1))
    for b in range(B):
        for tok in range(qo[b], qo[b + 1]):
            for head in range(hq):
                ranges = sorted(cover.pop((tok, head)))
                keys = np.zeros(int(kv_len[b]), dtype=int)
                for kv0, kv1 in ranges:
                    assert 0 <= kv0 <= kv1 <= kv_len[b]
                    keys[kv0:kv1] += 1
                assert np.all(keys == 1)
    assert not cover, "tiles cover rows that do not exist"
    _check_merge(p, g, hq)
    # the pool a run must hold: every listed page id below it
    assert p["raw"].kv_extent == (int(indices.max()) + 1 if indices.size else 0)


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("bs", [0, 1, 5, 128, 256])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (3, 1)])
def test_ragged_plan_covers_each_visible_pair_once(seed, bs, hq, hkv):
    rng = np.random.default_rng(seed + 7 * bs + hq)
    S = int(rng.integers(1, 5))
    lq = rng.integers(0, 300, S)
    cross = seed % 2 == 1 and bs == 0
    lk = rng.integers(0, 300, S) if cross else lq
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    p = plan_ragged_host(cu_q, cu_k if cross else None, bs, num_qo_heads=hq, num_kv_heads=hkv,
                         head_dim=128, num_sms=int(rng.integers(1, 5)))
    g = hq // hkv
    _check_cta_ptr(p)
    cover = {}
    for tok, head, kv0, kv1, i in _tiles_rows(p["tiles"], g):
        cover.setdefault((tok, head), []).append((kv0, kv1))
    for s in range(S):
        for tok in range(cu_q[s], cu_q[s + 1]):
            i_local = tok - cu_q[s]
            # visible keys by the definition, enumerated one by one
            vis = [j for j in range(int(lk[s])) if bs == 0 or (j // bs) <= (i_local // bs)]
            for head in range(hq):
                keys = np.zeros(int(lk[s]), dtype=int)
                for kv0, kv1 in cover.pop((tok, head)):
                    keys[kv0:kv1] += 1
                assert np.all(keys[vis] == 1), "a visible key is not covered exactly once"
                assert np.all(keys <= 1)
    assert not cover
    _check_merge(p, g, hq)
    assert p["raw"].kv_extent == int(cu_k[-1])       # key tokens a run's k and v must hold


def test_plan_is_deterministic():
    c = inputs.workload(3)
    kw = dict(num_qo_heads=32, num_kv_heads=8, head_dim=128, page_size=16)
    a = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages, **kw)
    b = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages, **kw)
    for k in ("header", "cta_ptr", "tiles"):
        assert np.array_equal(a[k], b[k])


def test_plan_balances_the_grid():
    c = inputs.workload(2)
    p = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages,
                        num_qo_heads=20, num_kv_heads=20, head_dim=64, page_size=16)
    t, cp = p["tiles"], p["cta_ptr"]
    load = np.array([int(((t[cp[i]:cp[i + 1], 5] - t[cp[i]:cp[i + 1], 4] + 15) // 16).sum() +
                         2 * (cp[i + 1] - cp[i])) for i in range(p["raw"].num_ctas)])
    assert p["raw"].num_ctas == 296
    assert load.max() <= 1.02 * load[:-1].mean() + 2


def test_workloads_choose_their_kernel_family():
    kinds = {}
    for i in (1, 2, 3, 5):
        c = inputs.workload(i)
        p = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len,
                            c.num_pages, num_qo_heads=c.num_qo_heads, num_kv_heads=c.num_kv_heads,
                            head_dim=c.head_dim, page_size=c.page_size)
        kinds[i] = p["raw"].kind
    # decode: CUDA-core kernel; 4 tokens x 8 heads at d=128: keys on the MMA M side;
    # up to 512 rows: 128-row query tiles
    assert kinds[1] == 1 and kinds[2] == 1 and kinds[3] == 2 and kinds[5] == 4


@pytest.mark.parametrize("mutate,match", [
    (lambda a: a.update(qo=np.array([0, 2, 1], np.int32)), "decreases"),
    (lambda a: a.update(qo=np.array([1, 2, 3], np.int32)), r"\[0\] must be 0"),
    (lambda a: a.update(idx=np.array([0, 1, 99], np.int32)), "outside"),
    (lambda a: a.update(idx=np.array([0, -1, 2], np.int32)), "outside"),
    (lambda a: a.update(kvl=np.array([16, 40], np.int32)), "fewer pages"),
    (lambda a: a.update(kvl=np.array([-1, 3], np.int32)), "kv_len < 0"),
])
def test_invalid_paged_inputs_are_rejected(mutate, match):
    a = dict(qo=np.array([0, 1, 2], np.int32), ip=np.array([0, 1, 3], np.int32),
             idx=np.array([0, 1, 2], np.int32), kvl=np.array([16, 20], np.int32))
    mutate(a)
    with pytest.raises(ValueError, match=match):
        plan_paged_host(a["qo"], a["ip"], a["idx"], a["kvl"], 4, num_qo_heads=4, num_kv_heads=2,
                        head_dim=64, page_size=16)


def test_unsupported_and_capacity_errors():
    with pytest.raises(ValueError, match="UNSUPPORTED|unsupported"):
        plan_paged_host([0, 1], [0, 1], [0], [3], 1, num_qo_heads=4, num_kv_heads=2, head_dim=96,
                        page_size=16)
    with pytest.raises(ValueError, match="CAPACITY"):
        plan_paged_host([0, 1, 2], [0, 1, 2], [0, 1], [3, 3], 2, num_qo_heads=4, num_kv_heads=2,
                        head_dim=64, page_size=16, max_batch=1)
    with pytest.raises(ValueError, match="CAPACITY"):
        plan_ragged_host([0, 300], None, 0, num_qo_heads=4, num_kv_heads=4, head_dim=64,
                         max_q_tokens=100)


def test_empty_inputs_plan_nothing():
    p = plan_paged_host([0], [0], [], [], 1, num_qo_heads=4, num_kv_heads=2, head_dim=64,
                        page_size=16)
    assert p["raw"].num_tiles == 0 and p["raw"].num_ctas == 0
    p = plan_paged_host([0, 0, 0], [0, 1, 2], [0, 1], [5, 9], 2, num_qo_heads=4, num_kv_heads=2,
                        head_dim=64, page_size=16)
    assert p["raw"].num_tiles == 0
    p = plan_ragged_host([0, 0], None, 4, num_qo_heads=2, num_kv_heads=2, head_dim=64)
    assert p["raw"].num_tiles == 0
    # a request with queries but no context keys gets one empty tile per unit (it writes
    # zeros); a decode unit holds both KV heads
    p = plan_paged_host([0, 2], [0, 0], [], [0], 1, num_qo_heads=4, num_kv_heads=2, head_dim=64,
                        page_size=16)
    t = p["tiles"]
    assert t.shape[0] == 1 and t[0, 10] == 2 and t[0, 4] == 0 and t[0, 5] == 0


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("hq,hkv,d,P", [(4, 2, 64, 16), (8, 1, 128, 32), (32, 8, 128, 16),
                                        (64, 8, 128, 64)])
def test_causal_paged_plan_covers_each_visible_pair_once(seed, hq, hkv, d, P):
    """Query i of a request (stream token kv_len - qlen + i) needs keys [0, kv_len - qlen + i]:
    each exactly once; keys past it may appear in its tile (the kernel masks them) but never
    twice, and no tile reaches past the unit's last query."""
    rng = np.random.default_rng(seed * 31 + hq)
    B = int(rng.integers(1, 6))
    kv_len = rng.integers(1, 700, B)
    q_len = np.minimum(kv_len, rng.integers(0, 90 if seed % 2 else 4, B))
    pages_per = (kv_len + P - 1) // P
    indptr = np.concatenate([[0], np.cumsum(pages_per)]).astype(np.int32)
    num_pages = int(indptr[-1]) + 3
    indices = rng.permutation(num_pages)[: indptr[-1]].astype(np.int32)
    qo = np.concatenate([[0], np.cumsum(q_len)]).astype(np.int32)
    p = plan_paged_host(qo, indptr, indices, kv_len, num_pages, num_qo_heads=hq,
                        num_kv_heads=hkv, head_dim=d, page_size=P,
                        num_sms=int(rng.integers(1, 9)), causal=True)
    assert p["raw"].kind in (1, 2) and p["header"][7] == 1
    g = hq // hkv
    _check_cta_ptr(p)
    cover = {}
    for tok, head, kv0, kv1, i in _tiles_rows(p["tiles"], g):
        cover.setdefault((tok, head), []).append((kv0, kv1))
    for b in range(B):
        for tok in range(qo[b], qo[b + 1]):
            lim = int(kv_len[b] - q_len[b] + (tok - qo[b]) + 1)
            for head in range(hq):
                keys = np.zeros(int(kv_len[b]), dtype=int)
                for kv0, kv1 in cover.pop((tok, head)):
                    assert 0 <= kv0 <= kv1 <= kv_len[b]
                    keys[kv0:kv1] += 1
                assert np.all(keys[:lim] == 1) and np.all(keys <= 1)
    assert not cover
    _check_merge(p, g, hq)


def test_causal_plan_rejects_more_queries_than_stream_tokens():
    with pytest.raises(ValueError, match="more queries"):
        plan_paged_host([0, 5], [0, 1], [0], [4], 1, num_qo_heads=4, num_kv_heads=2,
                        head_dim=64, page_size=16, causal=True)
    # the same arrays are fine for cross-attention
    plan_paged_host([0, 5], [0, 1], [0], [4], 1, num_qo_heads=4, num_kv_heads=2, head_dim=64,
                    page_size=16)


def test_causal_plan_trims_key_ranges_to_the_last_query():
    """A 64-token chunk at the start of a 4096-token stream needs only its first 64 keys."""
    qo = np.array([0, 64], np.int32)
    kv_len = np.array([64], np.int32)
    ip = np.array([0, 4], np.int32)
    p = plan_paged_host(qo, ip, np.arange(4, dtype=np.int32), kv_len, 4, num_qo_heads=32,
                        num_kv_heads=8, head_dim=128, page_size=16, causal=True)
    t = p["tiles"]
    assert p["raw"].kind == 2 and np.all(t[:, 5] <= 64)
    # 128 new tokens closing a 1128-token stream, GQA 4: units of 64 tokens (two 32-token
    # tiles); unit u's last query is stream token 1000 + 64 (u + 1) - 1
    qo = np.array([0, 128], np.int32)
    kv_len = np.array([1128], np.int32)
    ip = np.array([0, 71], np.int32)
    p = plan_paged_host(qo, ip, np.arange(71, dtype=np.int32), kv_len, 71, num_qo_heads=8,
                        num_kv_heads=2, head_dim=128, page_size=16, causal=True, num_sms=1)
    ends = sorted({(int(r[2]), int(r[5])) for r in p["tiles"]})
    assert ends == [(0, 1064), (64, 1128)]


@pytest.mark.parametrize("seed", range(4))
def test_tensor_core_plan_balances_block_steps(seed):
    """The tensor-core kernel spends about the same time on a key block whether the unit holds
    one 128-row query tile or two, so the plan balances block steps (plus one per tile): on
    block-causal spans of the benchmark's shape, with many one-tile span tails, the busiest
    CTA carries at most 4 % more steps than the mean."""
    rng = np.random.default_rng(seed)
    lens = []
    while sum(lens) < 65536:
        lens.append(int(rng.integers(256, 4097)))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    p = plan_ragged_host(cu, None, 256, num_qo_heads=16, num_kv_heads=16, head_dim=128)
    t, cp = p["tiles"], p["cta_ptr"]
    steps = [sum(-(-(int(t[i, 5]) - int(t[i, 4])) // 128) + 1 for i in range(cp[c], cp[c + 1]))
             for c in range(p["raw"].num_ctas)]
    assert max(steps) <= 1.04 * np.mean(steps), (max(steps), np.mean(steps))


def test_binding_rejects_buffers_of_the_wrong_shape():
    """The binding checks every device buffer's shape against the call before the library
    sees its pointer (the kernels read and write whole rows)."""
    import torch
    from ragged_attention_encoder_b200.api import _shape
    t = torch.zeros(5, 4, 64)
    _shape(t, "q", (5, 4, 64))
    _shape(t, "q", (None, 4, 64))
    for bad in [(4, 4, 64), (5, 2, 64), (5, 4, 128), (5, 4), (None, 4, 64, 1)]:
        with pytest.raises(ValueError, match="shape"):
            _shape(t, "q", bad)
    with pytest.raises(ValueError, match="tensor"):
        _shape(None, "q", (5, 4, 64))


def test_missing_library_fails_loudly():
    """Without the built library the binding raises: there is no CPU fallback."""
    import subprocess
    import sys
    code = ("import ragged_attention_encoder_b200._lib as L\n"
            "L.LIB_PATH = L.LIB_PATH + '.absent'\n"
            "L._lib = None\n"
            "try:\n"
            "    L.load()\n"
            "except ImportError as e:\n"
            "    print('raised', 'is missing' in str(e))\n")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=120)
    assert res.stdout.strip() == "raised True", res.stdout + res.stderr


def test_tensor_core_fill_does_not_overshoot_a_cta_by_a_block():
    """The contiguous fill closes a CTA when not one more key block fits in its capacity, so
    no CTA carries more than one block's cost above the mean (block costs 16 or 17, 16 per
    tile).  Few long units (2 requests x 8 KV heads over 30 000-key contexts) need that fill:
    whole units would leave most of the 148 CTAs idle."""
    case = inputs.paged_case(7, q_lens=[64, 40], ctx_lens=[30000, 21000], num_qo_heads=32,
                             num_kv_heads=8, head_dim=128, page_size=16)
    p = plan_paged_host(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices, case.kv_len,
                        case.num_pages, num_qo_heads=32, num_kv_heads=8, head_dim=128,
                        page_size=16, num_sms=148)
    assert p["raw"].kind == 2 and p["raw"].num_merge_rows > 0
    t, cp = p["tiles"], p["cta_ptr"]
    tpt = 128 // 4
    load = []
    for cta in range(p["raw"].num_ctas):
        s = 0
        for i in range(cp[cta], cp[cta + 1]):
            nb = -(-(int(t[i, 5]) - int(t[i, 4])) // 128)
            s += nb * (17 if int(t[i, 3]) > tpt else 16) + 16
        load.append(s)
    assert max(load) <= np.mean(load) + 17, (max(load), np.mean(load))


def test_tensor_core_plans_prefer_whole_units_when_balanced():
    """Whole units (no splits, a group's query chunks side by side) are chosen for the packed
    multi-token and chunked-prefill workloads, whose busiest CTA stays within 15 % of the
    split schedule's."""
    c = inputs.workload(3)
    p = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages,
                        num_qo_heads=32, num_kv_heads=8, head_dim=128, page_size=16)
    assert p["raw"].num_merge_rows == 0 and p["raw"].num_ctas == 148
    c = inputs.causal_chunked_prefill()
    p = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages,
                        num_qo_heads=c.num_qo_heads, num_kv_heads=c.num_kv_heads,
                        head_dim=c.head_dim, page_size=c.page_size, causal=True)
    assert p["raw"].num_merge_rows == 0 and p["raw"].num_ctas == 148
