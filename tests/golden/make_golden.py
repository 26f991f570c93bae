"""Writes the stored expected values under tests/golden/ by calling only the oracle.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from ragged_attention_encoder_b200 import inputs  # noqa: E402


def tiny_paged_decode():
    case = inputs.workload(1)
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    kp, vp = oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)
    out = oracle.paged_cross_attention(case.q, kp, vp, case.qo_indptr, case.kv_page_indptr,
                                       case.kv_page_indices, case.kv_len)
    return {"source": "oracle.paged_cross_attention on the tiny paged decode workload (seed 1)",
            "out": out.tolist(), "abs_sum": float(np.abs(out).sum())}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_paged_decode.json"), "w") as f:
        json.dump(tiny_paged_decode(), f)
    print("wrote tiny_paged_decode.json")
