"""Float64 reference for every step of the attention hot path -- TEST INFRASTRUCTURE ONLY.

What the path computes, written out as plainly as possible.  For each request (or span)
``r`` and query head ``h``::

    O[r, h] = softmax(Q[r, h] . K[r, kvh]^T * s  +  M) . V[r, kvh]

* ``s = 1/sqrt(head_dim)`` unless the caller gives another scale.
* ``kvh = h // (Hq / Hkv)``: contiguous groups of query heads share one KV head.  The M*
  model page (mstar.model.components.attention, ``Attention``) supports GQA by giving
  fewer KV heads than query heads; it does not spell out the head map, and contiguous
  groups are the reading taken here.
* ``M`` is 0 where a key is visible and -inf where it is not.  Softmax runs over keys,
  row by row, after subtracting the row maximum.  A row that sees no key at all yields
  zeros (the pages are silent on this case).

Visibility per path:

* Paged cross-attention (mstar.engine.resources.attn.cross, ``FlashInferCrossManager``):
  non-causal attention over an encoder context that was written once -- every query of
  request ``r`` sees all ``kv_len[r]`` context keys.  Keys are read from the pools
  through the page table: logical key ``t`` of request ``r`` lives in page
  ``kv_page_indices[kv_page_indptr[r] + t // P]`` at slot ``t % P``.
* Ragged block-causal self-attention (mstar.engine.resources.attn.ragged.base,
  ``RaggedBlockCausalAttnManager``): attention stays inside each span of one packed
  forward; positions are counted from the span start and grouped in blocks of
  ``block_size``; position ``i`` sees ``j`` iff ``j // bs <= i // bs``.
* Ragged two-span cross-attention (same page, ``RaggedCrossAttnManager``): the query
  span of request ``r`` sees every key of the request's key span, non-causally.
* Paged causal self-attention (mstar.engine.resources.attn.config, ``AttentionStep`` with
  ``causal=True``): the step's ``qlen`` queries are the last tokens of the request's
  ``kv_len``-token stream (their own K/V already appended); query ``i`` (0-based within the
  step) is token ``kv_len - qlen + i`` of the stream and sees keys ``0 .. kv_len - qlen + i``.
  The pages give only the flag; this position rule is the reading taken.

The inputs are exact bf16 values; they are upcast to float64 here, so the only error in
this module is float64 rounding.  Nothing here is blocked, fused or reordered.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def as_f64(x) -> np.ndarray:
    """Exact float64 copy of a bf16/fp32 torch tensor or an array-like."""
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _default_scale(head_dim: int, scale) -> float:
    if scale is None or scale <= 0:
        return 1.0 / math.sqrt(head_dim)
    return float(scale)


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                   visible: np.ndarray | None = None) -> np.ndarray:
    """softmax(q k^T * scale + mask) v for one head.

    q [n, d], k [L, d], v [L, d] (float64); ``visible`` is a boolean [n, L] mask (None:
    every key visible).  Rows without a visible key return zeros.
    """
    n, L = q.shape[0], k.shape[0]
    out = np.zeros((n, v.shape[1]), dtype=np.float64)
    if n == 0 or L == 0:
        return out
    scores = (q @ k.T) * scale
    if visible is None:
        visible = np.ones((n, L), dtype=bool)
    scores = np.where(visible, scores, -np.inf)
    row_max = scores.max(axis=1, keepdims=True)
    has_key = np.isfinite(row_max[:, 0])
    row_max = np.where(np.isfinite(row_max), row_max, 0.0)
    p = np.where(visible, np.exp(scores - row_max), 0.0)
    denom = p.sum(axis=1)
    num = p @ v
    out[has_key] = num[has_key] / denom[has_key, None]
    return out


def partial_attention_with_lse(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                               visible: np.ndarray | None = None):
    """Attention over a subset of keys plus its log-sum-exp (natural log).

    Returns (o [n, d], lse [n]); ``lse = log(sum_j exp(q.k_j * scale))`` over the visible
    keys, -inf for a row with none.  This is what one split of a split-KV schedule
    produces before the merge.
    """
    n, L = q.shape[0], k.shape[0]
    o = attention_rows(q, k, v, scale, visible)
    lse = np.full(n, -np.inf)
    if n == 0 or L == 0:
        return o, lse
    scores = (q @ k.T) * scale
    if visible is None:
        visible = np.ones((n, L), dtype=bool)
    scores = np.where(visible, scores, -np.inf)
    row_max = scores.max(axis=1)
    ok = np.isfinite(row_max)
    shifted = np.where(visible[ok], np.exp(scores[ok] - row_max[ok, None]), 0.0)
    lse[ok] = row_max[ok] + np.log(shifted.sum(axis=1))
    return o, lse


def merge_partials(o_parts: np.ndarray, lse_parts: np.ndarray) -> np.ndarray:
    """Split-KV merge: for partial outputs O_i with log-sum-exps lse_i,

    ``m = max_i lse_i``, ``w_i = exp(lse_i - m)``, ``O = sum_i w_i O_i / sum_i w_i``.
    o_parts [s, n, d], lse_parts [s, n] -> [n, d].  Rows whose every lse is -inf give 0.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    ok = np.isfinite(m)
    m_safe = np.where(ok, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe[None, :]), 0.0)
    num = (w[:, :, None] * o_parts).sum(axis=0)
    den = w.sum(axis=0)
    out = np.zeros(o_parts.shape[1:], dtype=np.float64)
    out[ok] = num[ok] / den[ok, None]
    return out


def block_causal_visible(length: int, block_size: int) -> np.ndarray:
    """[L, L] boolean mask of one span: i sees j iff j // bs <= i // bs (bs=0: all)."""
    i = np.arange(length)[:, None]
    j = np.arange(length)[None, :]
    if block_size <= 0:
        return np.ones((length, length), dtype=bool)
    return (j // block_size) <= (i // block_size)


def gather_paged_kv(pool, page_indptr, page_indices, request: int, kv_len: int) -> np.ndarray:
    """Logical K (or V) rows [kv_len, Hkv, d] of one request, read through its page list."""
    page_size = pool.shape[2]
    pages = np.asarray(page_indices)[int(page_indptr[request]):int(page_indptr[request + 1])]
    t = np.arange(int(kv_len))
    page_of, slot_of = pages[t // page_size], t % page_size
    if isinstance(pool, torch.Tensor):   # gather the bf16 rows, then upcast only those
        rows = pool[torch.from_numpy(page_of.astype(np.int64)), :,
                    torch.from_numpy(slot_of.astype(np.int64)), :]
        return as_f64(rows)
    return as_f64(pool)[page_of, :, slot_of, :]


def context_write(k_src: torch.Tensor, v_src: torch.Tensor, cu_enc, page_indptr, page_indices,
                  k_pool: torch.Tensor, v_pool: torch.Tensor):
    """Encode-step context write, done by plain element copies (bit exact).

    Token t of request b (row ``cu_enc[b] + t`` of the packed ``[sum_enc, Hkv, d]`` K/V)
    goes to page ``page_indices[page_indptr[b] + t // P]``, slot ``t % P`` of the pools
    ``[num_pages, Hkv, P, d]``.  Nothing else is touched.  Returns new pools.
    """
    k_out = k_pool.clone()
    v_out = v_pool.clone()
    page_size = k_pool.shape[2]
    for b in range(len(cu_enc) - 1):
        for t in range(int(cu_enc[b + 1]) - int(cu_enc[b])):
            page = int(page_indices[int(page_indptr[b]) + t // page_size])
            slot = t % page_size
            k_out[page, :, slot, :] = k_src[int(cu_enc[b]) + t]
            v_out[page, :, slot, :] = v_src[int(cu_enc[b]) + t]
    return k_out, v_out


def project_kv(hidden, w_k, b_k, w_v, b_v, num_kv_heads: int, head_dim: int):
    """K and V of the encoder context (mstar.model.components.attention,
    ``CrossAttention.compute_kv``): each packed encoder row ``x`` [hidden] goes through the K
    and V linears, ``k = x W_k^T (+ b_k)`` and ``v = x W_v^T (+ b_v)`` with nn.Linear weights
    ``[num_kv_heads * head_dim, hidden]``; float64; returned as [tokens, Hkv, d] each."""
    x = as_f64(hidden)
    k = x @ as_f64(w_k).T
    v = x @ as_f64(w_v).T
    if b_k is not None:
        k = k + as_f64(b_k)[None, :]
    if b_v is not None:
        v = v + as_f64(b_v)[None, :]
    return (k.reshape(x.shape[0], num_kv_heads, head_dim),
            v.reshape(x.shape[0], num_kv_heads, head_dim))


def append_kv(k_new: torch.Tensor, v_new: torch.Tensor, append_indptr, page_indptr,
              page_indices, kv_len, k_pool: torch.Tensor, v_pool: torch.Tensor):
    """Append of a step's own K/V to its stream, done by plain element copies (bit exact).

    The n = append_indptr[b+1] - append_indptr[b] new tokens of request b (rows
    ``append_indptr[b] + t`` of ``[sum_new, Hkv, d]``) are stream positions
    ``kv_len[b] - n + t`` (``kv_len`` counts the tokens after the append): page
    ``page_indices[page_indptr[b] + pos // P]``, slot ``pos % P``.  Returns new pools.
    """
    k_out = k_pool.clone()
    v_out = v_pool.clone()
    page_size = k_pool.shape[2]
    for b in range(len(append_indptr) - 1):
        n = int(append_indptr[b + 1]) - int(append_indptr[b])
        for t in range(n):
            pos = int(kv_len[b]) - n + t
            page = int(page_indices[int(page_indptr[b]) + pos // page_size])
            k_out[page, :, pos % page_size, :] = k_new[int(append_indptr[b]) + t]
            v_out[page, :, pos % page_size, :] = v_new[int(append_indptr[b]) + t]
    return k_out, v_out


def causal_append_visible(qlen: int, kv_len: int) -> np.ndarray:
    """[qlen, kv_len] boolean mask: query i (stream token kv_len - qlen + i) sees key j iff
    j <= kv_len - qlen + i."""
    i = np.arange(qlen)[:, None]
    j = np.arange(kv_len)[None, :]
    return j <= kv_len - qlen + i


def _kv_head(h: int, num_qo_heads: int, num_kv_heads: int) -> int:
    return h // (num_qo_heads // num_kv_heads)


def paged_cross_attention(q, k_pool, v_pool, qo_indptr, page_indptr, page_indices, kv_len,
                          scale=None) -> np.ndarray:
    """Non-causal cross-attention of packed queries over paged context K/V.

    q [sum_q, Hq, d]; pools [num_pages, Hkv, P, d]; returns float64 [sum_q, Hq, d].
    """
    qf = as_f64(q)
    hq, d = qf.shape[1], qf.shape[2]
    hkv = k_pool.shape[1]
    s = _default_scale(d, scale)
    out = np.zeros_like(qf)
    for b in range(len(kv_len)):
        q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        if q1 == q0:
            continue
        kb = gather_paged_kv(k_pool, page_indptr, page_indices, b, int(kv_len[b]))
        vb = gather_paged_kv(v_pool, page_indptr, page_indices, b, int(kv_len[b]))
        for h in range(hq):
            kvh = _kv_head(h, hq, hkv)
            out[q0:q1, h] = attention_rows(qf[q0:q1, h], kb[:, kvh], vb[:, kvh], s)
    return out


def paged_cross_attention_rows(q, k_pool, v_pool, qo_indptr, page_indptr, page_indices, kv_len,
                               rows, scale=None) -> np.ndarray:
    """The same as ``paged_cross_attention`` for selected (token, head) pairs only."""
    qo_indptr = np.asarray(qo_indptr)
    d = q.shape[2]
    hq, hkv = q.shape[1], k_pool.shape[1]
    s = _default_scale(d, scale)
    cache = {}
    out = np.zeros((len(rows), d))
    for n, (t, h) in enumerate(rows):
        b = int(np.searchsorted(qo_indptr, t, side="right") - 1)
        if b not in cache:
            cache[b] = (gather_paged_kv(k_pool, page_indptr, page_indices, b, int(kv_len[b])),
                        gather_paged_kv(v_pool, page_indptr, page_indices, b, int(kv_len[b])))
        kb, vb = cache[b]
        kvh = _kv_head(h, hq, hkv)
        qrow = as_f64(q[t, h])[None, :]
        out[n] = attention_rows(qrow, kb[:, kvh], vb[:, kvh], s)[0]
    return out


def paged_causal_attention(q, k_pool, v_pool, qo_indptr, page_indptr, page_indices, kv_len,
                           scale=None) -> np.ndarray:
    """Paged causal self-attention of each request's step queries over its stream.

    q [sum_q, Hq, d]; pools [num_pages, Hkv, P, d] holding each request's kv_len tokens;
    returns float64 [sum_q, Hq, d].
    """
    qf = as_f64(q)
    hq, d = qf.shape[1], qf.shape[2]
    hkv = k_pool.shape[1]
    s = _default_scale(d, scale)
    out = np.zeros_like(qf)
    for b in range(len(kv_len)):
        q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        if q1 == q0:
            continue
        kb = gather_paged_kv(k_pool, page_indptr, page_indices, b, int(kv_len[b]))
        vb = gather_paged_kv(v_pool, page_indptr, page_indices, b, int(kv_len[b]))
        vis = causal_append_visible(q1 - q0, int(kv_len[b]))
        for h in range(hq):
            kvh = _kv_head(h, hq, hkv)
            out[q0:q1, h] = attention_rows(qf[q0:q1, h], kb[:, kvh], vb[:, kvh], s, vis)
    return out


def paged_causal_attention_rows(q, k_pool, v_pool, qo_indptr, page_indptr, page_indices,
                                kv_len, rows, scale=None) -> np.ndarray:
    """The same as ``paged_causal_attention`` for selected (token, head) pairs only."""
    qo_indptr = np.asarray(qo_indptr)
    d = q.shape[2]
    hq, hkv = q.shape[1], k_pool.shape[1]
    s = _default_scale(d, scale)
    cache = {}
    out = np.zeros((len(rows), d))
    for n, (t, h) in enumerate(rows):
        b = int(np.searchsorted(qo_indptr, t, side="right") - 1)
        if b not in cache:
            cache[b] = (gather_paged_kv(k_pool, page_indptr, page_indices, b, int(kv_len[b])),
                        gather_paged_kv(v_pool, page_indptr, page_indices, b, int(kv_len[b])))
        kb, vb = cache[b]
        qlen = int(qo_indptr[b + 1]) - int(qo_indptr[b])
        vis = causal_append_visible(qlen, int(kv_len[b]))[t - int(qo_indptr[b])][None, :]
        out[n] = attention_rows(as_f64(q[t, h])[None, :], kb[:, _kv_head(h, hq, hkv)],
                                vb[:, _kv_head(h, hq, hkv)], s, vis)[0]
    return out


def ragged_block_causal_attention(q, k, v, cu_seqlens, block_size, scale=None) -> np.ndarray:
    """Cacheless block-causal self-attention within each span of a packed forward."""
    qf, kf, vf = as_f64(q), as_f64(k), as_f64(v)
    hq, d = qf.shape[1], qf.shape[2]
    hkv = kf.shape[1]
    s = _default_scale(d, scale)
    out = np.zeros_like(qf)
    for r in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[r]), int(cu_seqlens[r + 1])
        vis = block_causal_visible(b - a, block_size)
        for h in range(hq):
            kvh = _kv_head(h, hq, hkv)
            out[a:b, h] = attention_rows(qf[a:b, h], kf[a:b, kvh], vf[a:b, kvh], s, vis)
    return out


def ragged_block_causal_rows(q, k, v, cu_seqlens, block_size, rows, scale=None) -> np.ndarray:
    """The same as ``ragged_block_causal_attention`` for selected (token, head) pairs."""
    cu = np.asarray(cu_seqlens)
    d = q.shape[2]
    hq, hkv = q.shape[1], k.shape[1]
    s = _default_scale(d, scale)
    out = np.zeros((len(rows), d))
    for n, (t, h) in enumerate(rows):
        r = int(np.searchsorted(cu, t, side="right") - 1)
        a, b = int(cu[r]), int(cu[r + 1])
        i = t - a
        vis = block_causal_visible(b - a, block_size)[i][None, :]
        kvh = _kv_head(h, hq, hkv)
        out[n] = attention_rows(as_f64(q[t, h])[None, :], as_f64(k[a:b, kvh]),
                                as_f64(v[a:b, kvh]), s, vis)[0]
    return out


def ragged_cross_attention(q, k, v, cu_q, cu_kv, scale=None) -> np.ndarray:
    """Cacheless two-span cross-attention: query span r sees all of key span r."""
    qf, kf, vf = as_f64(q), as_f64(k), as_f64(v)
    hq, d = qf.shape[1], qf.shape[2]
    hkv = kf.shape[1]
    s = _default_scale(d, scale)
    out = np.zeros_like(qf)
    for r in range(len(cu_q) - 1):
        a, b = int(cu_q[r]), int(cu_q[r + 1])
        c, e = int(cu_kv[r]), int(cu_kv[r + 1])
        for h in range(hq):
            kvh = _kv_head(h, hq, hkv)
            out[a:b, h] = attention_rows(qf[a:b, h], kf[c:e, kvh], vf[c:e, kvh], s)
    return out
