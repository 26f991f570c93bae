"""The context write that needs no caller allocation, against the ordinary one.

Some callers cannot allocate device memory (their memory belongs to another allocator, or an
allocation is not allowed where they run), so they cannot hand the library a workspace.
rae_write_context_noalloc keeps its page-copy list in the library's own device array instead.
This file sorts last so that a run stopping at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from ragged_attention_encoder_b200 import Context, _lib, build, inputs

pytestmark = pytest.mark.gpu


def _p32(a):
    return a.ctypes.data_as(_lib.P32)


def _noalloc(lib, case, k, v, kp, vp):
    cu = np.ascontiguousarray(case.cu_enc, dtype=np.int32)
    ip = np.ascontiguousarray(case.kv_page_indptr, dtype=np.int32)
    ix = np.ascontiguousarray(case.kv_page_indices, dtype=np.int32)
    return lib.rae_write_context_noalloc(
        k.data_ptr(), v.data_ptr(), _p32(cu), _p32(ip), _p32(ix), int(case.batch), kp.data_ptr(),
        vp.data_ptr(), int(case.num_pages), case.num_kv_heads, case.head_dim, case.page_size,
        torch.cuda.current_stream().cuda_stream)


def test_no_alloc_context_write_matches_the_workspace_path():
    build.build()
    lib = _lib.load()
    cases = [
        inputs.paged_case(301, q_lens=[1] * 5, ctx_lens=(1, 900, 5), num_qo_heads=8,
                          num_kv_heads=4, head_dim=64, page_size=16, pool_pages=400),
        inputs.paged_case(302, q_lens=[1] * 3, ctx_lens=(1, 3000, 3), num_qo_heads=8,
                          num_kv_heads=2, head_dim=128, page_size=64, pool_pages=200),
    ]
    for case in cases:            # two calls in a row; the second reuses the library's array
        k, v = case.k_ctx.cuda(), case.v_ctx.cuda()
        shape = (case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
        kp = inputs.nan_pool(*shape, "cuda")
        vp = inputs.nan_pool(*shape, "cuda")
        assert _noalloc(lib, case, k, v, kp, vp) == _lib.RAE_OK
        ctx = Context(case.num_kv_heads, case.num_kv_heads, case.head_dim, case.page_size)
        rk = inputs.nan_pool(*shape, "cuda")
        rv = inputs.nan_pool(*shape, "cuda")
        ctx.write_context(k, v, case.cu_enc, case.kv_page_indptr, case.kv_page_indices, rk, rv)
        torch.cuda.synchronize()
        # byte work: the tolerance is bit equality
        assert torch.equal(kp.view(torch.int16), rk.view(torch.int16))
        assert torch.equal(vp.view(torch.int16), rv.view(torch.int16))


def test_no_alloc_context_write_rejects_more_pages_than_its_array():
    lib = _lib.load()
    n = 65537                                   # one page copy more than the array holds
    case = inputs.paged_case(303, q_lens=[1], ctx_lens=[1], num_qo_heads=1, num_kv_heads=1,
                             head_dim=64, page_size=16, pool_pages=4)
    case.cu_enc = np.array([0, n * 16], dtype=np.int32)
    case.kv_page_indptr = np.array([0, n], dtype=np.int32)
    case.kv_page_indices = np.arange(n, dtype=np.int32)
    case.num_pages = n
    kp = inputs.nan_pool(4, 1, 16, 64, "cuda")
    vp = inputs.nan_pool(4, 1, 16, 64, "cuda")
    k = torch.zeros(16, 1, 64, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, case, k, k, kp, vp) == _lib.RAE_ERR_CAPACITY
    assert b"65536" in lib.rae_last_error(None)     # the call has no context: per-thread message
    torch.cuda.synchronize()
    assert torch.all(kp.view(torch.int16) == inputs.BF16_NAN_BITS)


def test_no_alloc_context_write_refuses_a_capturing_stream():
    """The page list is copied from a host array that the next call rewrites, so a graph
    replaying that copy would write a later call's pages: under capture the call enqueues
    nothing and says why."""
    lib = _lib.load()
    case = inputs.paged_case(304, q_lens=[1, 1], ctx_lens=[40, 9], num_qo_heads=2,
                             num_kv_heads=2, head_dim=64, page_size=16, pool_pages=8)
    k, v = case.k_ctx.cuda(), case.v_ctx.cuda()
    shape = (case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    kp = inputs.nan_pool(*shape, "cuda")
    vp = inputs.nan_pool(*shape, "cuda")
    assert _noalloc(lib, case, k, v, kp, vp) == _lib.RAE_OK     # set-up outside any capture
    torch.cuda.synchronize()
    kp2 = inputs.nan_pool(*shape, "cuda")
    vp2 = inputs.nan_pool(*shape, "cuda")
    marker = torch.zeros(1, device="cuda")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        rc = _noalloc(lib, case, k, v, kp2, vp2)
        marker.add_(1)                           # so the captured graph is not empty
    assert rc == _lib.RAE_ERR_UNSUPPORTED
    assert b"capturing" in lib.rae_last_error(None)
    graph.replay()
    torch.cuda.synchronize()
    assert float(marker) == 1.0
    assert torch.all(kp2.view(torch.int16) == inputs.BF16_NAN_BITS)
    assert torch.all(vp2.view(torch.int16) == inputs.BF16_NAN_BITS)
    # the stream is usable afterwards and the call works again
    assert _noalloc(lib, case, k, v, kp2, vp2) == _lib.RAE_OK
    torch.cuda.synchronize()
    assert torch.equal(kp2.view(torch.int16), kp.view(torch.int16))
