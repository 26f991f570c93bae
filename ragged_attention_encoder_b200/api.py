"""Python binding of the C ABI (include/rae.h): argument marshalling only.

Every step of the attention path runs in the CUDA library; torch provides device memory and
the current stream.  Function and method names follow the C calls:

    ctx = Context(num_qo_heads=32, num_kv_heads=8, head_dim=128, page_size=16)
    ctx.write_context(k, v, cu_enc, page_indptr, page_indices, k_pool, v_pool)   # encode step
    plan = ctx.plan_paged(qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages)
    out = ctx.run_paged(plan, q, k_pool_layer, v_pool_layer)                     # per layer

``CrossAttention`` and ``RaggedAttention`` wrap a Context with the plan/run names of the M*
managers (FlashInferCrossManager, RaggedBlockCausalAttnManager, RaggedCrossAttnManager).
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib

__all__ = ["Context", "Plan", "CrossAttention", "RaggedAttention", "RaeError", "plan_paged_host",
           "plan_ragged_host"]


class RaeError(RuntimeError):
    """A CUDA or device-side failure reported by the library."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{_lib.STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _raise(status: int, message: str):
    if status in (_lib.RAE_ERR_INVALID_ARG, _lib.RAE_ERR_UNSUPPORTED, _lib.RAE_ERR_CAPACITY):
        raise ValueError(f"{_lib.STATUS_NAMES[status]}: {message}")
    raise RaeError(status, message)


def _i32(x) -> np.ndarray:
    """Host int32 array (contiguous) from a list, numpy array or CPU tensor."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr32(a: np.ndarray):
    return a.ctypes.data_as(_lib.P32)


def _shape(t: torch.Tensor, name: str, shape) -> None:
    """Raises unless t has len(shape) dimensions matching shape (None: any extent).  The
    library reads and writes whole rows of these buffers, so a short one must not reach it."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if t.dim() != len(shape) or any(e is not None and t.shape[i] != e for i, e in enumerate(shape)):
        want = ", ".join("*" if e is None else str(e) for e in shape)
        raise ValueError(f"{name} must have shape [{want}], got {list(t.shape)}")


def _dev(t: torch.Tensor, name: str, dtype=torch.bfloat16) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream_handle(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


class Plan:
    """An immutable, opaque plan (the C rae_plan plus the arrays it was built from)."""

    def __init__(self, raw: _lib.RaePlan, kind: str, num_pages: int = 0, total_kv: int = 0):
        self.raw = raw
        self.kind = kind
        self.num_pages = num_pages
        self.total_kv = total_kv

    @property
    def total_q(self) -> int:
        return self.raw.total_q

    @property
    def num_tiles(self) -> int:
        return self.raw.num_tiles

    @property
    def num_ctas(self) -> int:
        return self.raw.num_ctas

    @property
    def num_merge_rows(self) -> int:
        return self.raw.num_merge_rows

    @property
    def slot(self) -> int:
        return self.raw.slot

    @property
    def kernel_kind(self) -> int:
        return self.raw.kind


class Context:
    """One library context (geometry, capacities, two plan slots) plus its device workspace."""

    def __init__(self, num_qo_heads: int, num_kv_heads: int, head_dim: int, page_size: int = 16, *,
                 max_batch: int = 1024, max_q_tokens: int = 1 << 17, max_kv_pages: int = 1 << 18,
                 max_tiles: int = 1 << 16, max_partial_rows: int = 1 << 16, num_sms: int = 0,
                 device=None, library=None):
        # `library`: an already loaded build of the C library (the tests pass the hooked
        # test build); by default librae.so.
        self._lib = library if library is not None else _lib.load()
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        cfg = _lib.RaeConfig(num_qo_heads, num_kv_heads, head_dim, page_size, max_batch,
                             max_q_tokens, max_kv_pages, max_tiles, max_partial_rows, num_sms)
        self.config = cfg
        handle = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            st = self._lib.rae_create(ctypes.byref(handle), ctypes.byref(cfg))
        if st != _lib.RAE_OK:
            _raise(st, "rae_create failed (geometry, capacity or device not supported)")
        self._h = handle
        nbytes = int(self._lib.rae_workspace_bytes(self._h))
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self._next_slot = 0
        self.num_qo_heads = num_qo_heads
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        self.page_size = page_size

    # ------------------------------------------------------------------ plumbing
    def _check(self, st: int):
        if st != _lib.RAE_OK:
            msg = self._lib.rae_last_error(self._h)
            _raise(st, msg.decode() if msg else "")

    def _pools(self, k_pool, v_pool):
        _shape(k_pool, "k_pool", (None, self.num_kv_heads, self.page_size, self.head_dim))
        _shape(v_pool, "v_pool", tuple(k_pool.shape))

    def _tokens(self, t, name, rows, heads):
        _shape(t, name, (rows, heads, self.head_dim))

    def _slot(self, slot):
        if slot is None:
            slot = self._next_slot
            self._next_slot ^= 1
        return int(slot)

    def close(self):
        if getattr(self, "_h", None):
            self._lib.rae_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def workspace_bytes(self) -> int:
        return int(self.workspace.numel())

    def set_wait_timeout_ns(self, ns: int):
        self._check(self._lib.rae_set_wait_timeout_ns(self._h, int(ns)))

    def enable_kernel_timing(self, max_records: int):
        self._check(self._lib.rae_enable_kernel_timing(self._h, int(max_records)))

    def read_kernel_timing(self):
        """(attention-kernel ms, merge ms) of each run recorded since the last read; the split
        merge runs inside the attention kernel, so the second list holds zeros."""
        n_max = 1 << 16
        a = (ctypes.c_float * n_max)()
        m = (ctypes.c_float * n_max)()
        cnt = ctypes.c_int32()
        self._check(self._lib.rae_read_kernel_timing(self._h, a, m, n_max, ctypes.byref(cnt)))
        return list(a[:cnt.value]), list(m[:cnt.value])

    def check_device_status(self):
        self._check(self._lib.rae_check_device_status(self._h, self.workspace.data_ptr(),
                                                      _stream_handle(self.device)))

    # ------------------------------------------------------------------ calls
    def write_context(self, k_src, v_src, cu_enc, page_indptr, page_indices, k_pool, v_pool):
        cu = _i32(cu_enc)
        ip = _i32(page_indptr)
        ix = _i32(page_indices)
        batch = int(cu.shape[0] - 1)
        if ip.shape[0] != batch + 1:
            raise ValueError("page_indptr must have batch + 1 entries")
        n = int(cu[-1]) if batch > 0 else 0
        self._tokens(k_src, "k_src", n, self.num_kv_heads)
        self._tokens(v_src, "v_src", n, self.num_kv_heads)
        self._pools(k_pool, v_pool)
        self._check(self._lib.rae_write_context(
            self._h, _dev(k_src, "k_src"), _dev(v_src, "v_src"), _ptr32(cu), _ptr32(ip),
            _ptr32(ix) if ix.size else None, batch, _dev(k_pool, "k_pool"),
            _dev(v_pool, "v_pool"), int(k_pool.shape[0]), self.workspace.data_ptr(),
            _stream_handle(self.device)))

    def project_write_context(self, hidden, w_k, b_k, w_v, b_v, cu_enc, page_indptr,
                              page_indices, k_pool, v_pool):
        """Encode step with the K/V projections fused in: k = hidden . w_k^T (+ b_k) and
        v = hidden . w_v^T (+ b_v) for every packed token, stored straight into the pages.
        hidden [sum_enc, H]; w_k, w_v [Hkv * d, H] (nn.Linear layout); biases [Hkv * d] or
        None; all bf16 on the device."""
        cu = _i32(cu_enc)
        ip = _i32(page_indptr)
        ix = _i32(page_indices)
        batch = int(cu.shape[0] - 1)
        if ip.shape[0] != batch + 1:
            raise ValueError("page_indptr must have batch + 1 entries")
        n_out = self.num_kv_heads * self.head_dim
        if hidden.dim() != 2 or w_k.shape != (n_out, hidden.shape[1]) or w_v.shape != w_k.shape:
            raise ValueError("hidden must be [tokens, H] and w_k, w_v [num_kv_heads * head_dim, H]")
        if hidden.shape[0] != int(cu[-1]):
            raise ValueError("hidden must have cu_enc[-1] rows")
        self._pools(k_pool, v_pool)
        for b, name in ((b_k, "b_k"), (b_v, "b_v")):
            if b is not None and tuple(b.shape) != (n_out,):
                raise ValueError(f"{name} must have num_kv_heads * head_dim entries")
        self._check(self._lib.rae_project_write_context(
            self._h, _dev(hidden, "hidden"), int(hidden.shape[1]), _dev(w_k, "w_k"),
            None if b_k is None else _dev(b_k, "b_k"), _dev(w_v, "w_v"),
            None if b_v is None else _dev(b_v, "b_v"), _ptr32(cu), _ptr32(ip),
            _ptr32(ix) if ix.size else None, batch, _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
            int(k_pool.shape[0]), self.workspace.data_ptr(), _stream_handle(self.device)))

    def o_proj_partial(self, attn, w_o, bias=None, out=None):
        """One tensor-parallel rank's output projection: attn [m, Hq, d] (this context's heads,
        the run's output) or [m, Hq * d], times w_o [n, Hq * d] (the rank's columns of W_o,
        nn.Linear layout), plus bias [n] (bf16, or None); returns out [m, n] fp32.  The ranks'
        outputs sum to the full projection."""
        import torch
        m = int(attn.shape[0])
        k = self.num_qo_heads * self.head_dim
        if attn.numel() != m * k or attn.dtype != torch.bfloat16 or not attn.is_contiguous():
            raise ValueError("attn must be a contiguous bf16 [m, num_qo_heads, head_dim] tensor")
        if w_o.dim() != 2 or w_o.shape[1] != k or w_o.dtype != torch.bfloat16:
            raise ValueError("w_o must be bf16 [n, num_qo_heads * head_dim]")
        n = int(w_o.shape[0])
        if bias is not None and (tuple(bias.shape) != (n,) or bias.dtype != torch.bfloat16):
            raise ValueError("bias must be bf16 [n]")
        if out is None:
            out = torch.empty((m, n), dtype=torch.float32, device=self.device)
        elif tuple(out.shape) != (m, n) or out.dtype != torch.float32 or not out.is_contiguous():
            raise ValueError("out must be a contiguous fp32 [m, n] tensor")
        self._check(self._lib.rae_o_proj_partial(
            self._h, _dev(attn, "attn"), m, k, _dev(w_o, "w_o"), n,
            None if bias is None else _dev(bias, "bias"), _dev(out, "out", torch.float32),
            self.workspace.data_ptr(), _stream_handle(self.device)))
        return out

    def append_kv(self, k_new, v_new, append_indptr, kv_page_indptr, kv_page_indices, kv_len,
                  k_pool, v_pool):
        """Writes each request's new tokens (rows append_indptr[b]... of k_new / v_new) to the
        last positions of its kv_len[b]-token sequence (kv_len counts the appended tokens)."""
        ap = _i32(append_indptr)
        ip = _i32(kv_page_indptr)
        ix = _i32(kv_page_indices)
        kl = _i32(kv_len)
        batch = int(kl.shape[0])
        if ap.shape[0] != batch + 1 or ip.shape[0] != batch + 1:
            raise ValueError("append_indptr and kv_page_indptr must have batch + 1 entries")
        n = int(ap[-1]) if batch > 0 else 0
        self._tokens(k_new, "k_new", n, self.num_kv_heads)
        self._tokens(v_new, "v_new", n, self.num_kv_heads)
        self._pools(k_pool, v_pool)
        self._check(self._lib.rae_append_kv(
            self._h, _dev(k_new, "k_new"), _dev(v_new, "v_new"), _ptr32(ap), _ptr32(ip),
            _ptr32(ix) if ix.size else None, _ptr32(kl) if kl.size else None, batch,
            _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), int(k_pool.shape[0]),
            self.workspace.data_ptr(), _stream_handle(self.device)))

    def plan_paged(self, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages: int,
                   slot=None, causal: bool = False) -> Plan:
        """Plan of paged attention.  causal=False: cross-attention, every query sees all
        kv_len keys.  causal=True: the queries are the last tokens of each kv_len-token
        sequence and query i sees keys up to its own position, kv_len - qlen + i."""
        qo = _i32(qo_indptr)
        ip = _i32(kv_page_indptr)
        ix = _i32(kv_page_indices)
        kl = _i32(kv_len)
        batch = int(kl.shape[0])
        if qo.shape[0] != batch + 1 or ip.shape[0] != batch + 1:
            raise ValueError("qo_indptr and kv_page_indptr must have batch + 1 entries")
        raw = _lib.RaePlan()
        fn = self._lib.rae_plan_paged_causal if causal else self._lib.rae_plan_paged
        self._check(fn(
            self._h, self._slot(slot), _ptr32(qo), _ptr32(ip), _ptr32(ix) if ix.size else None,
            _ptr32(kl) if kl.size else None, batch, int(num_pages), self.workspace.data_ptr(),
            _stream_handle(self.device), ctypes.byref(raw)))
        return Plan(raw, "paged", num_pages=int(num_pages))

    def plan_ragged(self, cu_seqlens_q, cu_seqlens_kv=None, block_size: int = 0, slot=None) -> Plan:
        cq = _i32(cu_seqlens_q)
        ck = None if cu_seqlens_kv is None else _i32(cu_seqlens_kv)
        spans = int(cq.shape[0] - 1)
        if ck is not None and ck.shape[0] != spans + 1:
            raise ValueError("cu_seqlens_kv must have as many entries as cu_seqlens_q")
        raw = _lib.RaePlan()
        self._check(self._lib.rae_plan_ragged(
            self._h, self._slot(slot), _ptr32(cq), None if ck is None else _ptr32(ck), spans,
            int(block_size), self.workspace.data_ptr(), _stream_handle(self.device),
            ctypes.byref(raw)))
        total_kv = int((cq if ck is None else ck)[-1])
        return Plan(raw, "ragged", total_kv=total_kv)

    def run_paged(self, plan: Plan, q, k_pool, v_pool, out=None, sm_scale: float = 0.0):
        self._tokens(q, "q", plan.total_q, self.num_qo_heads)
        self._pools(k_pool, v_pool)
        if out is None:
            out = torch.empty_like(q)
        _shape(out, "out", tuple(q.shape))
        self._check(self._lib.rae_run_paged(
            self._h, ctypes.byref(plan.raw), _dev(q, "q"), _dev(k_pool, "k_pool"),
            _dev(v_pool, "v_pool"), int(k_pool.shape[0]), _dev(out, "out"), float(sm_scale),
            self.workspace.data_ptr(), _stream_handle(self.device)))
        return out

    def run_ragged(self, plan: Plan, q, k, v, out=None, sm_scale: float = 0.0):
        self._tokens(q, "q", plan.total_q, self.num_qo_heads)
        self._tokens(k, "k", None, self.num_kv_heads)
        _shape(v, "v", tuple(k.shape))
        if out is None:
            out = torch.empty_like(q)
        _shape(out, "out", tuple(q.shape))
        self._check(self._lib.rae_run_ragged(
            self._h, ctypes.byref(plan.raw), _dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
            int(k.shape[0]), _dev(out, "out"), float(sm_scale), self.workspace.data_ptr(),
            _stream_handle(self.device)))
        return out


class CrossAttention:
    """Paged cross-attention over a context written once (plan once per step, run per layer)."""

    def __init__(self, num_qo_heads: int, num_kv_heads: int, head_dim: int, page_size: int = 16,
                 **capacities):
        self.ctx = Context(num_qo_heads, num_kv_heads, head_dim, page_size, **capacities)

    def write_context(self, k, v, cu_enc, page_indptr, page_indices, k_pool, v_pool):
        self.ctx.write_context(k, v, cu_enc, page_indptr, page_indices, k_pool, v_pool)

    def plan(self, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages: int) -> Plan:
        return self.ctx.plan_paged(qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages)

    def run(self, q, k_pool, v_pool, plan: Plan, out=None, sm_scale: float = 0.0):
        return self.ctx.run_paged(plan, q, k_pool, v_pool, out, sm_scale)


class RaggedAttention:
    """Cacheless ragged attention: block-causal within spans, or two-span cross-attention."""

    def __init__(self, num_qo_heads: int, num_kv_heads: int, head_dim: int, **capacities):
        self.ctx = Context(num_qo_heads, num_kv_heads, head_dim, 16, **capacities)

    def plan(self, cu_seqlens_q, cu_seqlens_kv=None, block_size: int = 0) -> Plan:
        return self.ctx.plan_ragged(cu_seqlens_q, cu_seqlens_kv, block_size)

    def run(self, q, k, v, plan: Plan, out=None, sm_scale: float = 0.0):
        return self.ctx.run_ragged(plan, q, k, v, out, sm_scale)


# ---------------------------------------------------------------------- host-only planning

def _host_cfg(num_qo_heads, num_kv_heads, head_dim, page_size, num_sms, **cap):
    return _lib.RaeConfig(num_qo_heads, num_kv_heads, head_dim, page_size,
                          cap.get("max_batch", 1024), cap.get("max_q_tokens", 1 << 17),
                          cap.get("max_kv_pages", 1 << 18), cap.get("max_tiles", 1 << 16),
                          cap.get("max_partial_rows", 1 << 16), num_sms)


TILE_WORDS = 12   # {req, kv_head, q0, qn, kv0, kv1, part, split, munit, nsplit, pad, pad}


def _decode_image(img: np.ndarray, raw: _lib.RaePlan) -> dict:
    w = img.view(np.int32)
    n_ctas, n_tiles = raw.num_ctas, raw.num_tiles
    return {
        "header": w[:16].copy(),
        "cta_ptr": w[raw.off_cta_ptr:raw.off_cta_ptr + n_ctas + 1].copy() if n_ctas else
        np.zeros(1, np.int32),
        "tiles": w[raw.off_tiles:raw.off_tiles + TILE_WORDS * n_tiles].reshape(
            n_tiles, TILE_WORDS).copy(),
        "raw": raw,
    }


def plan_paged_host(qo_indptr, kv_page_indptr, kv_page_indices, kv_len, num_pages, *,
                    num_qo_heads, num_kv_heads, head_dim, page_size, num_sms=148, causal=False,
                    **cap) -> dict:
    """Runs the library's host plan builder without CUDA and decodes the plan image."""
    lib = _lib.load()
    cfg = _host_cfg(num_qo_heads, num_kv_heads, head_dim, page_size, num_sms, **cap)
    nbytes = int(lib.rae_plan_image_bytes_for(ctypes.byref(cfg)))
    if nbytes == 0:
        raise ValueError("unsupported configuration")
    img = np.zeros(nbytes, dtype=np.uint8)
    qo, ip, ix, kl = _i32(qo_indptr), _i32(kv_page_indptr), _i32(kv_page_indices), _i32(kv_len)
    raw = _lib.RaePlan()
    err = ctypes.create_string_buffer(512)
    fn = lib.rae_plan_paged_causal_host if causal else lib.rae_plan_paged_host
    st = fn(ctypes.byref(cfg), _ptr32(qo), _ptr32(ip),
                                 _ptr32(ix) if ix.size else None, _ptr32(kl) if kl.size else None,
                                 int(kl.shape[0]), int(num_pages), img.ctypes.data, nbytes,
                                 ctypes.byref(raw), err, 512)
    if st != _lib.RAE_OK:
        _raise(st, err.value.decode())
    return _decode_image(img, raw)


def plan_ragged_host(cu_seqlens_q, cu_seqlens_kv=None, block_size=0, *, num_qo_heads,
                     num_kv_heads, head_dim, num_sms=148, **cap) -> dict:
    lib = _lib.load()
    cfg = _host_cfg(num_qo_heads, num_kv_heads, head_dim, 16, num_sms, **cap)
    nbytes = int(lib.rae_plan_image_bytes_for(ctypes.byref(cfg)))
    if nbytes == 0:
        raise ValueError("unsupported configuration")
    img = np.zeros(nbytes, dtype=np.uint8)
    cq = _i32(cu_seqlens_q)
    ck = None if cu_seqlens_kv is None else _i32(cu_seqlens_kv)
    raw = _lib.RaePlan()
    err = ctypes.create_string_buffer(512)
    st = lib.rae_plan_ragged_host(ctypes.byref(cfg), _ptr32(cq), None if ck is None else _ptr32(ck),
                                  int(cq.shape[0] - 1), int(block_size), img.ctypes.data, nbytes,
                                  ctypes.byref(raw), err, 512)
    if st != _lib.RAE_OK:
        _raise(st, err.value.decode())
    return _decode_image(img, raw)
