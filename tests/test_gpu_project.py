"""Fused K/V projection and context write on the GPU, against the float64 oracle.

hidden [tokens, H] -> k = hidden . w_k^T (+ b_k), v = hidden . w_v^T (+ b_v), stored where
the context write stores each token.  Pools start as bf16 NaN: every slot the write must not
touch stays NaN, every slot it must write holds a finite value close to the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from ragged_attention_encoder_b200 import Context, inputs

from gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _inputs(seed, tokens, hidden, hkv, d, bias_k, bias_v):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(tokens, hidden, generator=g).to(torch.bfloat16)
    wk = (torch.randn(hkv * d, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    wv = (torch.randn(hkv * d, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    bk = torch.randn(hkv * d, generator=g).to(torch.bfloat16) if bias_k else None
    bv = torch.randn(hkv * d, generator=g).to(torch.bfloat16) if bias_v else None
    return x, wk, bk, wv, bv


def _check(case, kp, vp, k_ref, v_ref, what):
    """Written slots match the oracle; all other slots are still the NaN sentinel."""
    kp, vp = kp.cpu(), vp.cpu()
    got_k, got_v = [], []
    for b in range(case.batch):
        got_k.append(oracle.gather_paged_kv(kp, case.kv_page_indptr, case.kv_page_indices, b,
                                            int(case.kv_len[b])))
        got_v.append(oracle.gather_paged_kv(vp, case.kv_page_indptr, case.kv_page_indices, b,
                                            int(case.kv_len[b])))
    assert_close(np.concatenate(got_k), k_ref, what=f"{what} K")
    assert_close(np.concatenate(got_v), v_ref, what=f"{what} V")
    written = int(case.kv_len.sum()) * case.num_kv_heads * case.head_dim
    assert int((~torch.isnan(kp.float())).sum()) == written
    assert int((~torch.isnan(vp.float())).sum()) == written


@pytest.mark.parametrize("hidden,hkv,d,P,bias", [
    (1280, 20, 64, 16, (False, True)),     # the Whisper-large shape (k unbiased, v biased)
    (256, 2, 64, 16, (True, True)),
    (512, 8, 128, 64, (False, False)),
    (64, 4, 128, 32, (True, False)),
])
def test_projection_write_matches_oracle(hidden, hkv, d, P, bias):
    case = inputs.paged_case(400 + hidden + d + P, q_lens=[1, 1, 1, 1, 1],
                             ctx_lens=[1, 130, 17, 400, 255], num_qo_heads=hkv,
                             num_kv_heads=hkv, head_dim=d, page_size=P)
    x, wk, bk, wv, bv = _inputs(401 + hidden, int(case.cu_enc[-1]), hidden, hkv, d, *bias)
    ctx = Context(hkv, hkv, d, P)
    kp = inputs.nan_pool(case.num_pages, hkv, P, d, "cuda")
    vp = inputs.nan_pool(case.num_pages, hkv, P, d, "cuda")
    ctx.project_write_context(x.cuda(), wk.cuda(), None if bk is None else bk.cuda(), wv.cuda(),
                              None if bv is None else bv.cuda(), case.cu_enc, case.kv_page_indptr,
                              case.kv_page_indices, kp, vp)
    torch.cuda.synchronize()
    ctx.check_device_status()
    k_ref, v_ref = oracle.project_kv(x, wk, bk, wv, bv, hkv, d)
    _check(case, kp, vp, k_ref, v_ref, f"H={hidden} {hkv}x{d} P={P}")


def test_projection_rejects_unsupported_shapes():
    ctx = Context(3, 3, 64, 16)          # 3 * 64 = 192 output columns: not a multiple of 128
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(192, 64, dtype=torch.bfloat16, device="cuda")
    kp = inputs.nan_pool(2, 3, 16, 64, "cuda")
    with pytest.raises(ValueError, match="UNSUPPORTED"):
        ctx.project_write_context(x, w, None, w, None, [0, 4], [0, 1], [0], kp, kp.clone())


def test_whisper_encode_step_sampled():
    """The full Whisper-large encode step: 64 x 1500 tokens, hidden 1280, 20 x 64 heads,
    16 384-page pool; sampled tokens against the oracle and the NaN sentinel count."""
    case = inputs.workload(2)
    x, wk, bk, wv, bv = _inputs(410, int(case.cu_enc[-1]), 1280, 20, 64, False, True)
    ctx = Context(20, 20, 64, 16)
    kp = inputs.nan_pool(case.num_pages, 20, 16, 64, "cuda")
    vp = inputs.nan_pool(case.num_pages, 20, 16, 64, "cuda")
    ctx.project_write_context(x.cuda(), wk.cuda(), None, wv.cuda(), bv.cuda(), case.cu_enc,
                              case.kv_page_indptr, case.kv_page_indices, kp, vp)
    torch.cuda.synchronize()
    ctx.check_device_status()
    rng = np.random.default_rng(7)
    toks = np.unique(np.concatenate([rng.integers(0, int(case.cu_enc[-1]), 200),
                                     case.cu_enc[:-1], case.cu_enc[1:] - 1]))
    k_ref, v_ref = oracle.project_kv(x[toks], wk, bk, wv, bv, 20, 64)
    req = np.searchsorted(case.cu_enc, toks, side="right") - 1
    t_in = toks - case.cu_enc[req]
    pages = case.kv_page_indices[case.kv_page_indptr[req] + t_in // 16]
    slot = torch.from_numpy((t_in % 16).astype(np.int64))
    pg = torch.from_numpy(pages.astype(np.int64))
    got_k = kp[pg.cuda(), :, slot.cuda(), :].cpu()
    got_v = vp[pg.cuda(), :, slot.cuda(), :].cpu()
    assert_close(got_k, k_ref, what="whisper K rows")
    assert_close(got_v, v_ref, what="whisper V rows")
    written = int(case.cu_enc[-1]) * 20 * 64
    assert int((~torch.isnan(kp)).sum()) == written and int((~torch.isnan(vp)).sum()) == written
