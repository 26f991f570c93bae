"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's checks.

This module draws random numbers and lays out index arrays; it holds none of the
attention arithmetic (no products, no softmax, no page scatter).  It imports
nothing else from this package, so the CPU oracle's tests can use it without the
CUDA library.

Recipe (applied identically for every workload):

* ``torch.Generator('cpu').manual_seed(seed)``.
* Draw order: integer lengths, then the page permutation, then Q, then K, then V.
* Lengths are uniform and inclusive: ``randint(lo, hi + 1)``.
* Values are fp32 ``randn`` times a scale, rounded to bf16 (round to nearest even).
* A paged request ``b`` with context length ``n`` owns ``ceil(n / page_size)`` pages,
  taken in request order from a random permutation of the pool's page ids.

The five named workloads follow the shapes of the M* attention pages (paged
cross-attention over an encoder context written once, packed queries given by a
cumulative ``qo_indptr``, GQA through ``num_kv_heads < num_heads``, and cacheless
ragged block-causal attention within the spans of one packed forward).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC0  # quiet NaN used to poison untouched pool slots


@dataclass
class PagedCase:
    """One batch of paged cross-attention: packed queries over paged encoder K/V."""

    name: str
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int
    qo_indptr: np.ndarray          # int32 [B+1], cumulative query lengths
    kv_len: np.ndarray             # int32 [B], context length of each request
    kv_page_indptr: np.ndarray     # int32 [B+1]
    kv_page_indices: np.ndarray    # int32 [nnz], page ids in logical order
    cu_enc: np.ndarray             # int32 [B+1], cumulative context lengths (packed K/V rows)
    q: torch.Tensor                # bf16 [sum_q, Hq, d]
    k_ctx: torch.Tensor            # bf16 [sum_ctx, Hkv, d]  (packed compute_kv output)
    v_ctx: torch.Tensor            # bf16 [sum_ctx, Hkv, d]
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.kv_len.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.qo_indptr[-1])


@dataclass
class RaggedCase:
    """One packed forward of cacheless ragged attention (self or two-span cross)."""

    name: str
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int                # 0: no block mask (two-span cross); >0: block-causal
    cu_q: np.ndarray               # int32 [S+1]
    cu_kv: np.ndarray              # int32 [S+1]; equal to cu_q for self-attention
    q: torch.Tensor                # bf16 [Tq, Hq, d]
    k: torch.Tensor                # bf16 [Tkv, Hkv, d]
    v: torch.Tensor                # bf16 [Tkv, Hkv, d]
    self_attention: bool = True
    extra: dict = field(default_factory=dict)

    @property
    def num_spans(self) -> int:
        return int(self.cu_q.shape[0] - 1)


def _randint(g: torch.Generator, lo: int, hi: int, n: int) -> np.ndarray:
    if n == 0:
        return np.zeros(0, dtype=np.int32)
    return torch.randint(lo, hi + 1, (n,), generator=g).numpy().astype(np.int32)


def _bf16(g: torch.Generator, shape, scale: float) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16)


def _cumsum0(x: np.ndarray) -> np.ndarray:
    out = np.zeros(x.shape[0] + 1, dtype=np.int64)
    np.cumsum(x, out=out[1:])
    assert out[-1] < 2**31
    return out.astype(np.int32)


def paged_case(seed: int, *, q_lens, ctx_lens, num_qo_heads: int, num_kv_heads: int,
               head_dim: int, page_size: int, pool_pages=None, pool_factor: float = 1.25,
               scale: float = 1.0, name: str = "paged") -> PagedCase:
    """Draws a paged cross-attention batch.

    ``q_lens`` / ``ctx_lens`` are either a list of fixed lengths or a ``(lo, hi, B)``
    triple drawn uniformly (queries first, then contexts).  ``pool_pages`` fixes the
    pool size; otherwise it is ``ceil(pool_factor * pages_needed)``.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    # 1. lengths
    if isinstance(q_lens, tuple):
        lo, hi, b = q_lens
        q_len = _randint(g, lo, hi, b)
    else:
        q_len = np.asarray(q_lens, dtype=np.int32)
    if isinstance(ctx_lens, tuple):
        lo, hi, b = ctx_lens
        kv_len = _randint(g, lo, hi, b)
    else:
        kv_len = np.asarray(ctx_lens, dtype=np.int32)
    assert q_len.shape == kv_len.shape
    pages_per_req = (kv_len.astype(np.int64) + page_size - 1) // page_size
    kv_page_indptr = _cumsum0(pages_per_req)
    needed = int(kv_page_indptr[-1])
    num_pages = int(pool_pages) if pool_pages is not None else int(math.ceil(pool_factor * needed))
    num_pages = max(num_pages, needed, 1)
    # 2. page permutation
    perm = torch.randperm(num_pages, generator=g).numpy().astype(np.int32)
    kv_page_indices = np.ascontiguousarray(perm[:needed])
    qo_indptr = _cumsum0(q_len)
    cu_enc = _cumsum0(kv_len)
    # 3-5. Q, K, V
    q = _bf16(g, (int(qo_indptr[-1]), num_qo_heads, head_dim), scale)
    k_ctx = _bf16(g, (int(cu_enc[-1]), num_kv_heads, head_dim), scale)
    v_ctx = _bf16(g, (int(cu_enc[-1]), num_kv_heads, head_dim), scale)
    return PagedCase(name=name, num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads,
                     head_dim=head_dim, page_size=page_size, num_pages=num_pages,
                     qo_indptr=qo_indptr, kv_len=kv_len, kv_page_indptr=kv_page_indptr,
                     kv_page_indices=kv_page_indices, cu_enc=cu_enc, q=q, k_ctx=k_ctx, v_ctx=v_ctx)


def ragged_case(seed: int, *, span_lens=None, span_range=None, min_total: int = 0,
                kv_span_lens=None, num_qo_heads: int, num_kv_heads: int, head_dim: int,
                block_size: int, scale: float = 1.0, name: str = "ragged") -> RaggedCase:
    """Draws a packed forward of ragged spans.

    Either ``span_lens`` (fixed list) or ``span_range=(lo, hi)`` with spans drawn one at
    a time until their total reaches ``min_total`` (the last span is not trimmed).
    ``kv_span_lens`` (fixed list or ``(lo, hi)``) makes it a two-span cross-attention
    case: one key span per query span, drawn after the query spans.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    if span_lens is not None:
        q_spans = np.asarray(span_lens, dtype=np.int32)
    else:
        lo, hi = span_range
        lens = []
        total = 0
        while total < min_total:
            n = int(_randint(g, lo, hi, 1)[0])
            lens.append(n)
            total += n
        q_spans = np.asarray(lens, dtype=np.int32)
    self_attn = kv_span_lens is None
    if self_attn:
        kv_spans = q_spans
    elif isinstance(kv_span_lens, tuple):
        kv_spans = _randint(g, kv_span_lens[0], kv_span_lens[1], int(q_spans.shape[0]))
    else:
        kv_spans = np.asarray(kv_span_lens, dtype=np.int32)
    assert kv_spans.shape == q_spans.shape
    cu_q = _cumsum0(q_spans)
    cu_kv = _cumsum0(kv_spans)
    q = _bf16(g, (int(cu_q[-1]), num_qo_heads, head_dim), scale)
    k = _bf16(g, (int(cu_kv[-1]), num_kv_heads, head_dim), scale)
    v = _bf16(g, (int(cu_kv[-1]), num_kv_heads, head_dim), scale)
    return RaggedCase(name=name, num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads,
                      head_dim=head_dim, block_size=block_size, cu_q=cu_q, cu_kv=cu_kv,
                      q=q, k=k, v=v, self_attention=self_attn)


# ---------------------------------------------------------------------------------------
# The five named workloads.  The seed of workload i is i.

def tiny_paged_decode() -> PagedCase:
    """2 requests, 1 query token each, contexts 7 and 13, 4/2 heads, d=64, page 16, pool 8."""
    return paged_case(1, q_lens=[1, 1], ctx_lens=[7, 13], num_qo_heads=4, num_kv_heads=2,
                      head_dim=64, page_size=16, pool_pages=8, name="tiny_paged_decode")


def whisper_large_decode() -> PagedCase:
    """64 requests x 1 token over 1500-token contexts, 20/20 heads, d=64, page 16, 16384-page pool."""
    return paged_case(2, q_lens=[1] * 64, ctx_lens=[1500] * 64, num_qo_heads=20, num_kv_heads=20,
                      head_dim=64, page_size=16, pool_pages=16384, scale=0.5,
                      name="whisper_large_decode")


def packed_multitoken_cross() -> PagedCase:
    """32 requests, q ~ U[1,128], ctx ~ U[256,4096], 32/8 heads, d=128, page 16."""
    return paged_case(3, q_lens=(1, 128, 32), ctx_lens=(256, 4096, 32), num_qo_heads=32,
                      num_kv_heads=8, head_dim=128, page_size=16, name="packed_multitoken_cross")


def ragged_block_causal() -> RaggedCase:
    """Spans ~ U[256,4096] until >= 65536 tokens, block 256, 16/16 heads, d=128."""
    return ragged_case(4, span_range=(256, 4096), min_total=65536, num_qo_heads=16,
                       num_kv_heads=16, head_dim=128, block_size=256, name="ragged_block_causal")


def long_context_splitkv() -> PagedCase:
    """8 requests x 4 tokens, ctx ~ U[32768,131072], 64/8 heads, d=128, page 64."""
    return paged_case(5, q_lens=[4] * 8, ctx_lens=(32768, 131072, 8), num_qo_heads=64,
                      num_kv_heads=8, head_dim=128, page_size=64, name="long_context_splitkv")


WORKLOADS = {
    1: tiny_paged_decode,
    2: whisper_large_decode,
    3: packed_multitoken_cross,
    4: ragged_block_causal,
    5: long_context_splitkv,
}


def causal_chunked_prefill() -> PagedCase:
    """Paged causal self-attention, chunked prefill: 32 requests each append a 128-token
    chunk that closes a stream of U[256, 4096] tokens (the chunk included); 32 query heads /
    8 KV heads, head_dim 128, pages of 16 tokens, bf16 N(0,1), random page table."""
    return paged_case(6, q_lens=[128] * 32, ctx_lens=(256, 4096, 32), num_qo_heads=32,
                      num_kv_heads=8, head_dim=128, page_size=16,
                      name="paged_causal_chunked_prefill")


def workload(i: int):
    return WORKLOADS[i]()


def nan_pool(num_pages: int, num_kv_heads: int, page_size: int, head_dim: int,
             device="cpu") -> torch.Tensor:
    """A K or V pool [num_pages, Hkv, P, d] whose every slot holds a bf16 NaN."""
    bits = torch.full((num_pages, num_kv_heads, page_size, head_dim), BF16_NAN_BITS,
                      dtype=torch.int16, device=device)
    return bits.view(torch.bfloat16)
