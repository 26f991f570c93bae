#!/usr/bin/env python
"""Benchmark of the attention hot path on B200; prints ONE JSON line (rank 0).

Headline workload: the Whisper-large-shaped decoder cross-attention decode step -- 64 requests
x 1 query token over 1500-token encoder contexts, 20/20 heads, head_dim 64, pages of 16 tokens
scattered over a 16384-page pool.  One step is what a decoder step of that model does with
this path: one plan (host, once per step) and then one layer call per decoder layer (32),
each layer reading its own layer's context pool.  All pools stay resident in HBM (32 x 2 x
671 MB); every layer's 491.5 MB of valid K/V exceeds the 126 MB L2, so nothing is served
from L2 between layers.

  value  KV HBM GB/s of the whole step: algorithmic bytes (valid K/V once per KV head + Q + O)
         over the device time of K steps (CUDA events, max over ranks), uninstrumented.
  roofline  the decode kernel's bytes per launch over its mean launch duration, from CUDA
         events the library records around each kernel in a second pass of the same K steps.
  e2e    the same metric through the public API with host buffers: every layer's q is copied
         host->device from pinned memory and every output back, inside the timed region.

The other four workloads (tiny decode, packed multi-token, ragged block-causal, long-context
split-KV) are measured per layer call under "workloads".  `--impl reference` times the CPU
float64 oracle (the only reference this path has) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

LAYERS = 32                       # decoder layers of the Whisper-large shape
SPEC_TC_TFLOPS = 2250.0           # dense bf16 per B200 (nominal)
SPEC_HBM_GBS = 8000.0             # HBM3e per B200 (nominal)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-workloads", action="store_true",
                    help="only the headline workload (no per-workload table)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile-case", type=int, default=None, choices=[1, 2, 3, 4, 5, 6, 7],
                    help="run only this workload's layer call --reps times (for ncu captures); "
                         "6: paged causal chunked prefill, 7: the fused K/V projection")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--tp", action="store_true",
                    help="tensor-parallel: the decode step's heads sharded over the --gpus ranks, "
                         "each layer's o_proj partial summed by one all-reduce (strong scaling)")
    ap.add_argument("--counters", action="store_true",
                    help="capture the ncu counters of every workload's kernel (one launch each, "
                         "a few metrics) and write them to --counters-out; prints no benchmark line")
    ap.add_argument("--counters-out", default=None,
                    help="file the counters go to (default profiles/counters.json)")
    return ap.parse_args()


# ---------------------------------------------------------------------- work accounting

def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks (x itself outside a process group).  Every rank calls it
    at the same point: it is one collective."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput of replicas: every rank processes the same bytes per step, and the
    step takes the slowest rank's time."""
    return bytes_per_rank_step * world / (ms_per_step * 1e-3) / 1e9


def paged_work(case, causal=False):
    """(flops, bytes) of one layer call: 4*d*Hq per visible (query, key) pair; valid K/V read
    once per KV head, plus Q and O.  Causal: query i of a request sees kv_len - qlen + i + 1
    keys."""
    q_len = np.diff(case.qo_indptr).astype(np.int64)
    kv = case.kv_len.astype(np.int64)
    if causal:
        pairs = int((q_len * (kv - q_len) + q_len * (q_len + 1) // 2).sum())
    else:
        pairs = int((q_len * kv).sum())
    flops = 4 * case.head_dim * case.num_qo_heads * pairs
    kv_tokens = int(kv[q_len > 0].sum())
    kv_bytes = kv_tokens * case.num_kv_heads * case.head_dim * 2 * 2
    qo_bytes = int(q_len.sum()) * case.num_qo_heads * case.head_dim * 2 * 2
    return flops, kv_bytes + qo_bytes, kv_bytes


def ragged_work(case):
    pairs = 0
    for s in range(case.num_spans):
        lq = int(case.cu_q[s + 1] - case.cu_q[s])
        lk = int(case.cu_kv[s + 1] - case.cu_kv[s])
        if case.block_size > 0:
            i = np.arange(lq, dtype=np.int64)
            pairs += int(np.minimum(lk, (i // case.block_size + 1) * case.block_size).sum())
        else:
            pairs += lq * lk
    flops = 4 * case.head_dim * case.num_qo_heads * pairs
    kv_bytes = int(case.cu_kv[-1]) * case.num_kv_heads * case.head_dim * 2 * 2
    qo_bytes = int(case.cu_q[-1]) * case.num_qo_heads * case.head_dim * 2 * 2
    return flops, kv_bytes + qo_bytes, kv_bytes


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "tflops": float(p["bf16_tflops"]),
                "tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "tflops": FALLBACK_TFLOPS,
                "tflops_sustained": 1400.0, "source": "fallback"}


# Kernel of each workload's layer call, and the sources it is built from.
PROFILE_CASES = {
    1: ("tiny_paged_decode", "decode_simt_kernel", "decode_simt.cu"),
    2: ("whisper_large_decode", "decode_simt_kernel", "decode_simt.cu"),
    3: ("packed_multitoken_cross", "attn_tc_kernel", "attn_tc.cu"),
    4: ("ragged_block_causal", "attn_tc_kernel", "attn_tc.cu"),
    5: ("long_context_splitkv", "attn_swapab_kernel", "attn_swapab.cu"),
    6: ("paged_causal_chunked_prefill", "attn_tc_kernel", "attn_tc.cu"),
    7: ("whisper_encode_kv_projection_write", "project_write_kernel", "project_write.cu"),
}
COUNTER_METRICS = ("gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum,"
                   "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed,"
                   "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed")
COUNTERS_PATH = os.path.join(ROOT, "profiles", "counters.json")


def kernel_source_sha(source: str) -> str:
    """Hash of a kernel's .cu file and every header of the library's sources: counters are
    only reported for the source they were taken on."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "ragged_attention_encoder_b200", "csrc")
    h = hashlib.sha256()
    files = [os.path.join(csrc, source)] + sorted(
        glob.glob(os.path.join(csrc, "*.cuh")) + glob.glob(os.path.join(csrc, "*.h")))
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_counters(workload: str):
    """The ncu counters of the workload's kernel from profiles/counters.json, if they were
    taken on the current source (else None)."""
    try:
        with open(COUNTERS_PATH) as f:
            entries = json.load(f)
    except Exception:
        return None
    for e in entries:
        if e.get("workload") != workload:
            continue
        try:
            if kernel_source_sha(e["source"]) != e.get("source_sha"):
                return None
        except Exception:
            return None
        return e
    return None


def load_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the workload's kernel, from the counters."""
    e = load_counters(workload)
    return None if e is None else float(e["dram_bytes_read"] + e["dram_bytes_write"])


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.15)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for name, flag in zip(names, r[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------- our arm

def flush_l2(buf):
    """Evicts the timed call's inputs from L2: writes the first half of `buf` (2 x 256 MB, each
    half twice the 126 MB L2), then reads the second half, which also evicts -- and writes
    back, before the timed region -- the dirty lines the write left, so the timed call neither
    hits L2 nor pays for another buffer's write-back."""
    half = buf.numel() // 2
    buf[:half].zero_()
    buf[half:].max()


def time_layer_calls(ctx, calls, warmup, reps, flush_buf):
    """Kernel time (attention + merge, ms) per call: CUDA events recorded by the library
    around its kernels on the launching stream, L2 flushed before every call."""
    import torch
    for _ in range(warmup):
        calls()
    torch.cuda.synchronize()
    ctx.enable_kernel_timing(reps)
    for _ in range(reps):
        flush_l2(flush_buf)
        calls()
    torch.cuda.synchronize()
    attn, merge = ctx.read_kernel_timing()
    ctx.enable_kernel_timing(0)
    return [a + m for a, m in zip(attn, merge)], attn, merge


def setup_workload(i, dev):
    """One workload's context, plan and layer call on `dev`: (case, ctx, plan, call, flops,
    bytes, host plan µs).  Paged workloads get their context through the context write."""
    import torch
    from ragged_attention_encoder_b200 import Context, inputs
    causal = i == 6
    case = inputs.causal_chunked_prefill() if causal else inputs.workload(i)
    if hasattr(case, "kv_page_indices"):
        ctx = Context(case.num_qo_heads, case.num_kv_heads, case.head_dim, case.page_size,
                      device=dev)
        kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, dev)
        vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, dev)
        ctx.write_context(case.k_ctx.to(dev), case.v_ctx.to(dev), case.cu_enc,
                          case.kv_page_indptr, case.kv_page_indices, kp, vp)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        plan = ctx.plan_paged(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices,
                              case.kv_len, case.num_pages, causal=causal)
        plan_us = (time.perf_counter() - t0) * 1e6
        q = case.q.to(dev)
        out = torch.empty_like(q)
        call = lambda: ctx.run_paged(plan, q, kp, vp, out)  # noqa: E731
        flops, nbytes, _ = paged_work(case, causal)
    else:
        ctx = Context(case.num_qo_heads, case.num_kv_heads, case.head_dim, 16, device=dev)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        plan = ctx.plan_ragged(case.cu_q, None, case.block_size)
        plan_us = (time.perf_counter() - t0) * 1e6
        q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
        out = torch.empty_like(q)
        call = lambda: ctx.run_ragged(plan, q, k, v, out)  # noqa: E731
        flops, nbytes, _ = ragged_work(case)
    return case, ctx, plan, call, flops, nbytes, plan_us


def projection_setup(dev):
    """Inputs of the Whisper-large encode step with fused K/V projection; returns the call."""
    import torch
    from ragged_attention_encoder_b200 import Context, inputs
    case = inputs.workload(2)
    m, hidden, hkv, d = int(case.cu_enc[-1]), 1280, 20, 64
    gen = torch.Generator(device=dev).manual_seed(77)
    x = torch.randn(m, hidden, generator=gen, device=dev).to(torch.bfloat16)
    wk = (torch.randn(hkv * d, hidden, generator=gen, device=dev) / hidden ** 0.5).to(torch.bfloat16)
    wv = (torch.randn(hkv * d, hidden, generator=gen, device=dev) / hidden ** 0.5).to(torch.bfloat16)
    bv = torch.randn(hkv * d, generator=gen, device=dev).to(torch.bfloat16)
    ctx = Context(hkv, hkv, d, 16, device=dev)
    kp = torch.empty(case.num_pages, hkv, 16, d, dtype=torch.bfloat16, device=dev)
    vp = torch.empty_like(kp)

    def fused():
        ctx.project_write_context(x, wk, None, wv, bv, case.cu_enc, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)
    return case, ctx, x, wk, wv, bv, kp, vp, fused


def projection_row(dev, peaks, flush_buf):
    """The Whisper-large encode step with the K/V projections fused into the context write:
    64 x 1500 encoder tokens, hidden 1280, 20 KV heads x 64 (k unbiased, v biased), seeded
    random weights; CUDA events around each call (median of 30 after 5 warm-ups, L2 flushed),
    next to the unfused sequence (two torch linears, then the context write)."""
    import torch
    import torch.nn.functional as F
    case, ctx, x, wk, wv, bv, kp, vp, fused = projection_setup(dev)
    m, hkv, d = int(case.cu_enc[-1]), 20, 64
    hidden = x.shape[1]

    def unfused():
        k = F.linear(x, wk).view(m, hkv, d)
        v = F.linear(x, wv, bv).view(m, hkv, d)
        ctx.write_context(k, v, case.cu_enc, case.kv_page_indptr, case.kv_page_indices, kp, vp)

    def timed(fn):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ts = []
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(30):
            flush_l2(flush_buf)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts) * 1e-3
    t = timed(fused)
    ctx.check_device_status()
    t_unfused = timed(unfused)
    flops = 2 * m * hidden * 2 * hkv * d
    nbytes = m * hidden * 2 + 2 * hkv * d * hidden * 2 + 2 * m * hkv * d * 2
    tc = flops / t / 1e12
    return {
        "us_per_call": round(t * 1e6, 2),
        "tflops": round(tc, 1),
        "hbm_gbs": round(nbytes / t / 1e9, 1),
        "bound": "tensor",
        "tc_frac_of_measured": round(tc / peaks["tflops"], 4),
        "tc_frac_of_measured_sustained": round(tc / peaks["tflops_sustained"], 4),
        "tc_frac_of_spec": round(tc / SPEC_TC_TFLOPS, 4),
        "algorithmic_flops": flops,
        "algorithmic_bytes": nbytes,
        "unfused_us": round(t_unfused * 1e6, 2),
        "unfused": "torch F.linear (cuBLAS) for K and V, then the library's context write",
    }


def q_projection_row(i, dev, flush_buf):
    """The Q projection in front of a layer call (page "mstar.model.components.attention",
    CrossAttention: q = h . W_q^T + b_q, projected every step; hidden = Hq * d, seeded
    synthetic weights): the cuBLAS GEMM and the run in sequence, against the run alone, with
    what fusing the GEMM into the run's Q load could save at most (the q tensor's write and
    read at the measured HBM peak, plus one launch).  Median of 30 calls, L2 flushed."""
    import torch
    import torch.nn.functional as F
    case, ctx, plan, call, _, _, _ = setup_workload(i, dev)
    tokens = int(case.qo_indptr[-1])
    hidden = case.num_qo_heads * case.head_dim
    gen = torch.Generator(device=dev).manual_seed(90 + i)
    h = torch.randn(tokens, hidden, generator=gen, device=dev).to(torch.bfloat16)
    w_q = (torch.randn(hidden, hidden, generator=gen, device=dev) / hidden ** 0.5).to(torch.bfloat16)
    b_q = torch.randn(hidden, generator=gen, device=dev).to(torch.bfloat16)
    q = case.q.to(dev)

    def gemm():
        q.copy_(F.linear(h, w_q, b_q).view_as(q))

    def timed(fn):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(30):
            flush_l2(flush_buf)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(ts)

    t_run = timed(call)
    t_gemm = timed(lambda: F.linear(h, w_q, b_q))
    t_both = timed(lambda: (gemm(), call()))
    ctx.check_device_status()
    q_bytes = tokens * hidden * 2
    del ctx
    return {"tokens": tokens, "hidden": hidden, "run_us": round(t_run, 2),
            "q_gemm_us": round(t_gemm, 2), "gemm_then_run_us": round(t_both, 2),
            "fusion_saves_at_most_us": round(2 * q_bytes / (6550.0 * 1e9) * 1e6 + 2.0, 2),
            "note": "the bound counts q written and read once at 6550 GB/s plus 2 us of launch"}


def counters_row(workload: str, algorithmic_bytes: int):
    """ncu counters of the row's kernel (one launch, cold L2) taken on the current source, or
    None: DRAM traffic per launch against the algorithmic bytes, tensor-pipe and DRAM
    utilisation."""
    e = load_counters(workload)
    if e is None:
        return None
    traffic = e["dram_bytes_read"] + e["dram_bytes_write"]
    return {"kernel": e["kernel"], "traffic": traffic,
            "traffic_over_algorithmic": round(traffic / algorithmic_bytes, 3),
            "tensor_pipe_pct": e["tensor_pipe_pct"], "dram_throughput_pct": e["dram_throughput_pct"],
            "ncu_time_us": e["gpu_time_us"], "source_sha": e["source_sha"]}


def workload_table(dev, peaks, flush_buf):
    """Per-layer-call numbers of the five workloads, and of paged causal chunked prefill (6):
    median of 100 calls after 10 warm-up calls, L2 flushed before every call (a 256 MB
    write, then a 256 MB read that writes its dirty lines back)."""
    import torch
    rows = {}
    for i in (1, 2, 3, 4, 5, 6):
        case, ctx, plan, call, flops, nbytes, plan_us = setup_workload(i, dev)
        tot, attn, merge = time_layer_calls(ctx, call, 10, 100, flush_buf)
        ctx.check_device_status()
        t = statistics.median(tot) * 1e-3
        ta = statistics.median(attn) * 1e-3
        tc = flops / t / 1e12
        gbs = nbytes / t / 1e9
        t_star_spec = max(flops / (SPEC_TC_TFLOPS * 1e12), nbytes / (SPEC_HBM_GBS * 1e9))
        t_star_meas = max(flops / (peaks["tflops"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
        bound = "tensor" if flops / (SPEC_TC_TFLOPS * 1e12) > nbytes / (SPEC_HBM_GBS * 1e9) else "hbm"
        rows[case.name] = {
            "us_per_layer_call": round(t * 1e6, 2),
            "attention_kernel_us": round(ta * 1e6, 2),
            "merge_us": round(statistics.median(merge) * 1e3, 2),
            "tflops": round(tc, 2),
            "hbm_gbs": round(gbs, 1),
            "bound": bound,
            "roofline_frac_of_spec": round(t_star_spec / t, 4),
            "roofline_frac_of_measured": round(t_star_meas / t, 4),
            "tc_frac_of_spec": round(tc / SPEC_TC_TFLOPS, 4),
            "tc_frac_of_measured": round(tc / peaks["tflops"], 4),
            "tc_frac_of_measured_sustained": round(tc / peaks["tflops_sustained"], 4),
            "hbm_frac_of_measured": round(gbs / peaks["hbm_gbs"], 4),
            "hbm_frac_of_spec": round(gbs / SPEC_HBM_GBS, 4),
            "algorithmic_flops": flops,
            "algorithmic_bytes": nbytes,
            "tiles": plan.num_tiles,
            "ctas": plan.num_ctas,
            "merge_rows": plan.num_merge_rows,
            "plan_host_us": round(plan_us, 1),
            "counters": counters_row(case.name, nbytes),
        }
        del ctx
        torch.cuda.empty_cache()
    rows["q_projection_then_run"] = {
        "whisper_large_decode": q_projection_row(2, dev, flush_buf),
        "packed_multitoken_cross": q_projection_row(3, dev, flush_buf)}
    torch.cuda.empty_cache()
    rows["whisper_encode_kv_projection_write"] = projection_row(dev, peaks, flush_buf)
    rows["whisper_encode_kv_projection_write"]["counters"] = counters_row(
        "whisper_encode_kv_projection_write",
        rows["whisper_encode_kv_projection_write"]["algorithmic_bytes"])
    torch.cuda.empty_cache()
    return rows


def cpu_oracle_rate(case, budget_s):
    """The float64 oracle on the host cores, repeated over the workload's requests for about
    budget_s seconds; returns (GB/s of the same algorithmic bytes, seconds, requests)."""
    import oracle
    from ragged_attention_encoder_b200 import inputs
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    kp, vp = oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)
    _, nbytes, _ = paged_work(case)
    per_req = nbytes / case.batch
    done, t0 = 0, time.perf_counter()
    b = 0
    while True:
        qo = case.qo_indptr
        sub_q = case.q[qo[b]:qo[b + 1]]
        oracle.paged_cross_attention(sub_q, kp, vp, np.array([0, qo[b + 1] - qo[b]]),
                                     case.kv_page_indptr[b:b + 2] - case.kv_page_indptr[b],
                                     case.kv_page_indices[case.kv_page_indptr[b]:],
                                     case.kv_len[b:b + 1])
        done += 1
        b = (b + 1) % case.batch
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return per_req * done / el / 1e9, el, done


def cpu_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        blas = None
    return n, blas


def run_ours(args):
    import torch
    import torch.distributed as dist
    from ragged_attention_encoder_b200 import Context, inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks = load_peaks()

    case = inputs.workload(2)
    flops, nbytes, kv_bytes = paged_work(case)
    ctx = Context(case.num_qo_heads, case.num_kv_heads, case.head_dim, case.page_size, device=dev)

    # Layer 0 gets the seeded context through the library's context write (timed as a1);
    # layers 1..31 get seeded random pools drawn on the device.
    k_pools, v_pools, qs, outs = [], [], [], []
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, dev)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim, dev)
    k_src, v_src = case.k_ctx.to(dev), case.v_ctx.to(dev)
    ctx.write_context(k_src, v_src, case.cu_enc, case.kv_page_indptr, case.kv_page_indices, kp, vp)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # One call alone (the host builds the page list while the device waits), and the steady
    # state of calls back to back, as an encode step writes its layers (the host work of one
    # call overlaps the device's work on the previous one).
    wtimes, btimes = [], []
    burst = 4
    for _ in range(5):
        e0.record()
        ctx.write_context(k_src, v_src, case.cu_enc, case.kv_page_indptr, case.kv_page_indices, kp, vp)
        e1.record()
        torch.cuda.synchronize()
        wtimes.append(e0.elapsed_time(e1))
        e0.record()
        for _ in range(burst):
            ctx.write_context(k_src, v_src, case.cu_enc, case.kv_page_indptr, case.kv_page_indices,
                              kp, vp)
        e1.record()
        torch.cuda.synchronize()
        btimes.append(e0.elapsed_time(e1) / burst)
    write_bytes = 2 * 2 * int(case.cu_enc[-1]) * case.num_kv_heads * case.head_dim * 2
    write_ms = statistics.median(wtimes)
    write_burst_ms = statistics.median(btimes)
    del k_src, v_src
    k_pools.append(kp)
    v_pools.append(vp)
    qs.append(case.q.to(dev))
    gen = torch.Generator(device=dev).manual_seed(1000 + rank)
    shape = (case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    for _ in range(1, LAYERS):
        k_pools.append(torch.randn(shape, generator=gen, device=dev, dtype=torch.bfloat16))
        v_pools.append(torch.randn(shape, generator=gen, device=dev, dtype=torch.bfloat16))
        qs.append(torch.randn(case.q.shape, generator=gen, device=dev, dtype=torch.bfloat16))
    outs = [torch.empty_like(q) for q in qs]

    def step():
        plan = ctx.plan_paged(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices,
                              case.kv_len, case.num_pages)
        for layer in range(LAYERS):
            ctx.run_paged(plan, qs[layer], k_pools[layer], v_pools[layer], outs[layer])
        return plan

    plan = step()
    for _ in range(max(args.warmup - 1, 0)):
        step()
    torch.cuda.synchronize()
    ctx.check_device_status()

    # ---------------------------------------------------------------- timed region
    # The step exactly as a user runs it: no per-kernel events (they serialise the launches).
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        step()
    t_end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    dev_ms = t_start.elapsed_time(t_end)
    ctx.check_device_status()
    dev_ms = max_over_ranks(dev_ms, dev)

    # ---------------------------------------------------------------- kernel-timed region
    # The same K steps again with the library recording CUDA events around each attention
    # kernel on its stream: the per-launch durations behind the roofline.
    ctx.enable_kernel_timing(args.steps * LAYERS)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    attn_ms, merge_ms = ctx.read_kernel_timing()
    ctx.enable_kernel_timing(0)
    ctx.check_device_status()
    ms_per_step = dev_ms / args.steps
    step_bytes = nbytes * LAYERS
    value = job_gbs(step_bytes, world, ms_per_step)

    # ---------------------------------------------------------------- end to end
    # Through the public API with host buffers: every step's 32 query tensors come from pinned
    # host memory and its 32 outputs go back to it, inside the timed region.  As a serving loop
    # would, the copies run on a second stream, double-buffered, so that step i+1's inputs and
    # step i's outputs move while step i+1 / step i compute.
    q_host = torch.empty((LAYERS,) + tuple(case.q.shape), dtype=torch.bfloat16, pin_memory=True)
    for layer, q in enumerate(qs):
        q_host[layer].copy_(q)
    o_host = torch.empty(q_host.shape, dtype=torch.bfloat16, pin_memory=True)
    q_dev = [torch.empty(q_host.shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    o_dev = [torch.empty(q_host.shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    copy_stream = torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(1, min(args.steps, 50))

    def e2e_run(n, start_event=None):
        with torch.cuda.stream(copy_stream):
            if start_event is not None:
                copy_stream.wait_event(start_event)
            q_dev[0].copy_(q_host, non_blocking=True)
            in_ready[0].record(copy_stream)
        p = None
        for i in range(n):
            b = i % 2
            comp.wait_event(in_ready[b])
            p = ctx.plan_paged(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices,
                               case.kv_len, case.num_pages)
            for layer in range(LAYERS):
                ctx.run_paged(p, q_dev[b][layer], k_pools[layer], v_pools[layer], o_dev[b][layer])
            done[b].record(comp)
            with torch.cuda.stream(copy_stream):
                if i + 1 < n:
                    if i >= 1:
                        copy_stream.wait_event(done[b ^ 1])   # step i-1 has read q_dev[b ^ 1]
                    q_dev[b ^ 1].copy_(q_host, non_blocking=True)
                    in_ready[b ^ 1].record(copy_stream)
                copy_stream.wait_event(done[b])
                o_host.copy_(o_dev[b], non_blocking=True)
        comp.wait_stream(copy_stream)
        return p

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_start.record(comp)
    p = e2e_run(e2e_steps, t_start)
    t_end.record(comp)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ctx.check_device_status()
    if not torch.equal(o_host[0], outs[0].cpu()):
        raise RuntimeError("end-to-end output differs from the device-timed run")
    e2e_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    e2e_value = job_gbs(step_bytes, world, e2e_ms / e2e_steps)
    h2d = int(q_host.numel()) * 2 + p.raw.image_words * 4
    d2h = int(o_host.numel()) * 2

    # ---------------------------------------------------------------- roofline (decode kernel)
    attn_mean_ms = statistics.fmean(attn_ms) if attn_ms else float("nan")
    launch_bytes = nbytes                        # one layer call's algorithmic bytes
    achieved = launch_bytes / (attn_mean_ms * 1e-3) / 1e9
    traffic = load_traffic("whisper_large_decode")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "kernel": "decode_simt_kernel<64,1>",
                "peak_source": peaks["source"],
                "frac_of_spec_8TBs": round(achieved / SPEC_HBM_GBS, 4)}

    result = {
        "metric": "KV HBM GB/s per B200 (Whisper-large decode cross-attention step: plan + 32 layer calls)",
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; layer 0 from the CPU generator, layers 1-31 device-seeded)",
        "config": {"workload": "whisper_large_decode", "requests": 64, "q_tokens_per_request": 1,
                   "context_tokens": 1500, "num_qo_heads": 20, "num_kv_heads": 20,
                   "head_dim": 64, "page_size": 16, "pool_pages": 16384,
                   "layers_per_step": LAYERS, "l2": "inputs larger than L2 (491.5 MB K/V per layer)",
                   "parallelism": f"replicas x{world}"},
        "us_per_layer_call": round(ms_per_step * 1e3 / LAYERS, 2),
        "attention_kernel_us": round(attn_mean_ms * 1e3, 2),
        "merge_kernel_us": round(statistics.fmean(merge_ms) * 1e3, 2) if merge_ms else 0.0,
        "tflops": round(flops * LAYERS * world / (ms_per_step * 1e-3) / 1e12, 3),
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms / e2e_steps, 4),
                "copies": "pinned host <-> device on a second stream, double-buffered"},
        "gpu_launches": int(len(attn_ms) + sum(1 for m in merge_ms if m > 0)),
        "clocks": clocks,
        "plan": {"tiles": plan.num_tiles, "ctas": plan.num_ctas, "merge_rows": plan.num_merge_rows},
        "context_write": {"gbs": round(write_bytes / (write_ms * 1e-3) / 1e9, 1),
                          "ms": round(write_ms, 4), "bytes": write_bytes,
                          "back_to_back_gbs": round(write_bytes / (write_burst_ms * 1e-3) / 1e9, 1),
                          "back_to_back_ms": round(write_burst_ms, 4),
                          "note": "read + write bytes; one call alone (host page-list work "
                                  "exposed), and calls back to back"},
    }

    if world == 1 and rank == 0:
        gbs, secs, reqs = cpu_oracle_rate(case, args.cpu_seconds)
        cores, blas = cpu_cores()
        result["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                  "blas_threads": blas, "kind": "oracle",
                                  "sample": f"float64 oracle over {reqs} request-layer calls of "
                                            f"the workload ({secs:.1f} s)"}
    del k_pools, v_pools
    torch.cuda.empty_cache()
    if world == 1 and not args.skip_workloads:
        flush = torch.zeros(512 << 20, dtype=torch.uint8, device=dev)
        result["workloads"] = workload_table(dev, peaks, flush)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------- tensor-parallel arm

def run_tp(args):
    """The Whisper-large decode step with its 20 heads sharded over the ranks (page
    "mstar.model.components.distributed.attention", ParallelAttention): every rank plans and
    runs its heads of each of the 32 layers, multiplies its attention output by its columns of
    W_o (hidden 1280, synthetic seeded weights; rank 0 adds the bias) and takes part in one fp32
    all-reduce per layer.  Total work is fixed as N grows (strong scaling); value counts the
    unsharded layer's KV bytes per step over the slowest rank's device time."""
    import datetime

    import torch
    import torch.distributed as dist
    from ragged_attention_encoder_b200 import inputs
    from ragged_attention_encoder_b200.tp import TensorParallelCrossAttention

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    case = inputs.workload(2)
    hidden = case.num_qo_heads * case.head_dim          # Whisper-large: 1280
    tp = TensorParallelCrossAttention(case.num_qo_heads, case.num_kv_heads, case.head_dim,
                                      case.page_size, rank=rank, world=world, device=dev)
    s = tp.shard
    gen = torch.Generator(device=dev).manual_seed(2000 + rank)
    shape = (case.num_pages, s.num_kv_heads, case.page_size, case.head_dim)
    k_pools, v_pools, qs, ws, outs, projs = [], [], [], [], [], []
    for _ in range(LAYERS):
        k_pools.append(torch.randn(shape, generator=gen, device=dev, dtype=torch.bfloat16))
        v_pools.append(torch.randn(shape, generator=gen, device=dev, dtype=torch.bfloat16))
        qs.append(torch.randn((case.q.shape[0], s.num_qo_heads, case.head_dim), generator=gen,
                              device=dev, dtype=torch.bfloat16))
        ws.append((torch.randn((hidden, s.num_qo_heads * case.head_dim), generator=gen, device=dev)
                   / hidden ** 0.5).to(torch.bfloat16))
        outs.append(torch.empty_like(qs[-1]))
        projs.append(torch.empty((case.q.shape[0], hidden), dtype=torch.float32, device=dev))
    b_o = torch.randn(hidden, generator=gen, device=dev).to(torch.bfloat16)

    def step():
        plan = tp.plan(case.qo_indptr, case.kv_page_indptr, case.kv_page_indices, case.kv_len,
                       case.num_pages)
        for layer in range(LAYERS):
            tp.forward(plan, qs[layer], k_pools[layer], v_pools[layer], ws[layer], b_o,
                       outs[layer], projs[layer])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    tp.ctx.check_device_status()
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    tp.ctx.check_device_status()
    ms = max_over_ranks(t0.elapsed_time(t1), dev) / args.steps
    flops, nbytes, _ = paged_work(case)
    tokens = int(case.qo_indptr[-1])
    proj_flops = 2 * tokens * hidden * hidden
    value = nbytes * LAYERS / (ms * 1e-3) / 1e9
    result = {
        "metric": "KV HBM GB/s (Whisper-large decode cross-attention step with o_proj, heads "
                  "sharded over the GPUs)",
        "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (device-seeded pools, queries and W_o)",
        "config": {"workload": "whisper_large_decode_tp", "requests": 64, "context_tokens": 1500,
                   "num_qo_heads": 20, "num_kv_heads": 20, "head_dim": 64, "page_size": 16,
                   "hidden": hidden, "layers_per_step": LAYERS,
                   "heads_per_rank": s.num_qo_heads, "parallelism": f"tp{world}",
                   "collective": "one fp32 all-reduce of [64, 1280] per layer (NCCL)"},
        "us_per_layer_call": round(ms * 1e3 / LAYERS, 2),
        "o_proj_tflop_per_step": round(proj_flops * LAYERS / 1e12, 4),
        "gpu_launches": 2 * LAYERS * args.steps,
        "clocks": clocks,
        "e2e": None,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from ragged_attention_encoder_b200 import inputs
    import oracle
    case = inputs.workload(2)
    _, nbytes, _ = paged_work(case)
    per_req = nbytes / case.batch
    kp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    vp = inputs.nan_pool(case.num_pages, case.num_kv_heads, case.page_size, case.head_dim)
    kp, vp = oracle.context_write(case.k_ctx, case.v_ctx, case.cu_enc, case.kv_page_indptr,
                                  case.kv_page_indices, kp, vp)

    def one(b):   # one request of one layer call: the bounded sample of a step
        qo = case.qo_indptr
        oracle.paged_cross_attention(case.q[qo[b]:qo[b + 1]], kp, vp, np.array([0, 1]),
                                     case.kv_page_indptr[b:b + 2] - case.kv_page_indptr[b],
                                     case.kv_page_indices[case.kv_page_indptr[b]:],
                                     case.kv_len[b:b + 1])

    for w in range(args.warmup):
        one(w % case.batch)
    t0 = time.perf_counter()
    for s in range(args.steps):
        one(s % case.batch)
    el = time.perf_counter() - t0
    value = per_req * args.steps / el / 1e9
    cores, blas = cpu_cores()
    ms = el / args.steps * 1e3
    print(json.dumps({
        "impl": "reference",
        "metric": "KV HBM GB/s per B200 (Whisper-large decode cross-attention step: plan + 32 layer calls)",
        "value": round(value, 5), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": "whisper_large_decode", "requests": 64, "q_tokens_per_request": 1,
                   "context_tokens": 1500, "num_qo_heads": 20, "num_kv_heads": 20, "head_dim": 64,
                   "page_size": 16, "pool_pages": 16384, "layers_per_step": LAYERS,
                   "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": cores,
                         "blas_threads": blas, "kind": "oracle",
                         "sample": "each step: the float64 oracle on one request of one layer call"},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_profile_case(args):
    """`--profile-case I --reps N`: workload I's layer call N times and nothing else (the
    command that ncu captures run; it prints no benchmark line)."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.profile_case == 7:
        case, ctx, *_, call = projection_setup(dev)
        info = {"profile_case": "whisper_encode_kv_projection_write"}
    else:
        case, ctx, plan, call, _, _, _ = setup_workload(args.profile_case, dev)
        info = {"profile_case": case.name, "kind": plan.kernel_kind, "tiles": plan.num_tiles,
                "ctas": plan.num_ctas}
    for _ in range(args.reps):
        call()
    torch.cuda.synchronize()
    ctx.check_device_status()
    print(json.dumps({**info, "reps": args.reps}), flush=True)


def _ncu_csv_metrics(path: str):
    """{metric: value} of the single launch in an ncu --csv log (units as ncu prints them)."""
    import csv
    with open(path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    out = {}
    for row in csv.DictReader(lines):
        name, unit, val = row.get("Metric Name"), row.get("Metric Unit", ""), row.get("Metric Value")
        if not name or val is None:
            continue
        v = float(val.replace(",", ""))
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "nsecond": 1e-3,
                 "ns": 1e-3, "usecond": 1.0, "us": 1.0, "msecond": 1e3, "ms": 1e3,
                 "%": 1.0}.get(unit, 1.0)
        out[name] = v * scale
    return out


def run_counters(args):
    """ncu counters of every workload's kernel: each `--profile-case I` command runs once
    plainly, then under ncu with a handful of metrics on one launch (the second of its
    kernel; `--clock-control none`).  Writes profiles/counters.json."""
    ncu = os.environ.get("NCU", "ncu")
    outdir = os.environ.get("RAE_NCU_LOG_DIR") or tempfile.mkdtemp()   # raw ncu CSVs
    os.makedirs(outdir, exist_ok=True)
    entries = []
    for case_id, (workload, kernel, source) in PROFILE_CASES.items():
        cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--profile-case", str(case_id),
               "--reps", "3"]
        plain = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
        if plain.returncode != 0:
            raise RuntimeError(f"profile case {case_id} failed without ncu:\n{plain.stderr[-2000:]}")
        log = os.path.join(outdir, f"counters_{workload}.csv")
        ncmd = [ncu, "--metrics", COUNTER_METRICS, "--clock-control", "none", "-k",
                f"regex:{kernel}", "-s", "1", "-c", "1", "--csv", "--log-file", log] + cmd
        t0 = time.time()
        res = subprocess.run(ncmd, capture_output=True, text=True, timeout=900)
        if res.returncode != 0:
            raise RuntimeError(f"ncu on case {case_id} failed:\n{res.stdout[-2000:]}\n{res.stderr[-2000:]}")
        m = _ncu_csv_metrics(log)
        entries.append({
            "workload": workload, "kernel": kernel, "source": source,
            "source_sha": kernel_source_sha(source),
            "gpu_time_us": round(m["gpu__time_duration.sum"], 2),
            "dram_bytes_read": int(m["dram__bytes_read.sum"]),
            "dram_bytes_write": int(m["dram__bytes_write.sum"]),
            "tensor_pipe_pct": round(m["sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed"], 2),
            "dram_throughput_pct": round(m["gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed"], 2),
            "command": " ".join(["ncu", "--metrics", COUNTER_METRICS, "--clock-control", "none",
                                 "-k", f"regex:{kernel}", "-s", "1", "-c", "1", "python", "bench.py",
                                 "--profile-case", str(case_id), "--reps", "3"]),
            "capture_s": round(time.time() - t0, 1),
        })
        print(json.dumps(entries[-1]), flush=True)
    with open(args.counters_out or COUNTERS_PATH, "w") as f:
        json.dump(entries, f, indent=1)
        f.write("\n")


def main():
    args = parse()
    if args.counters:
        run_counters(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_case is not None:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.tp:
        run_tp(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
