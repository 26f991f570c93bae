"""Helpers of the GPU tests: run a workload through the C-ABI and compare with the oracle."""
import numpy as np
import torch

import oracle
from ragged_attention_encoder_b200 import Context, inputs

ATOL = 2e-2        # max-abs error bound on bf16 outputs
REL_L2 = 5e-3      # ||gpu - ref||_2 / ||ref||_2 bound


def assert_close(out, ref, atol=ATOL, rel_l2=REL_L2, what=""):
    g = out.detach().float().cpu().numpy().astype(np.float64) if isinstance(out, torch.Tensor) \
        else np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = float(np.abs(g - ref).max()) if g.size else 0.0
    nref = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref)) / nref if nref > 0 else float(np.linalg.norm(g))
    assert err <= atol and rel <= rel_l2, f"{what}: max-abs {err:.3e}, rel-L2 {rel:.3e}"
    return err, rel


def context_for(case, **cap):
    return Context(case.num_qo_heads, case.num_kv_heads, case.head_dim,
                   getattr(case, "page_size", 16), **cap)


def gpu_pools(case, ctx):
    """NaN-filled pools on the device, then the context write through the library."""
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, "cuda")
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, "cuda")
    ctx.write_context(case.k_ctx.cuda(), case.v_ctx.cuda(), case.cu_enc, case.kv_page_indptr,
                      case.kv_page_indices, kp, vp)
    return kp, vp


def oracle_pools(case):
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    return oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                case.kv_page_indices, kp, vp)


def run_paged(case, ctx=None, sm_scale=0.0, **cap):
    ctx = ctx or context_for(case, **cap)
    kp, vp = gpu_pools(case, ctx)
    plan = ctx.plan_paged(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices, case.kv_len,
                          case.num_pages)
    q = case.q.cuda()
    out = torch.full_like(q, float("nan"))
    ctx.run_paged(plan, q, kp, vp, out, sm_scale)
    torch.cuda.synchronize()
    ctx.check_device_status()
    return out, plan, ctx, kp, vp


def run_ragged(case, ctx=None, sm_scale=0.0, **cap):
    ctx = ctx or Context(case.num_qo_heads, case.num_kv_heads, case.head_dim, 16, **cap)
    plan = ctx.plan_ragged(case.cu_q, None if case.self_attention else case.cu_kv, case.block_size)
    q, k, v = case.q.cuda(), case.k.cuda(), case.v.cuda()
    out = torch.full_like(q, float("nan"))
    ctx.run_ragged(plan, q, k, v, out, sm_scale)
    torch.cuda.synchronize()
    ctx.check_device_status()
    return out, plan, ctx


def oracle_paged(case, scale=None):
    kp, vp = oracle_pools(case)
    return oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                        case.kv_page_indices, case.kv_len, scale)


def oracle_ragged(case, scale=None):
    if case.self_attention:
        return oracle.ragged_block_causal_attention(case.q, case.k, case.v, case.cu_q,
                                                    case.block_size, scale)
    return oracle.ragged_cross_attention(case.q, case.k, case.v, case.cu_q, case.cu_kv, scale)
