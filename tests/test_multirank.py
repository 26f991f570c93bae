"""The N > 1 host path on CPU: two gloo ranks, as `bench.py --gpus 2` runs them.

The path shards as replicas (each rank runs the whole decode step on its own GPU; no tensor
crosses ranks), so what needs checking is host logic: every rank builds the identical plan
from the same seeded workload, the step time is the maximum over ranks, the whole-job value
counts every rank's bytes, and the reference arm prints from rank 0 alone.
"""
import hashlib
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _plan_digest(workload: int) -> str:
    from ragged_attention_encoder_b200 import inputs, plan_paged_host
    c = inputs.workload(workload)
    p = plan_paged_host(c.qo_indptr, c.kv_page_indptr, c.kv_page_indices, c.kv_len, c.num_pages,
                        num_qo_heads=c.num_qo_heads, num_kv_heads=c.num_kv_heads,
                        head_dim=c.head_dim, page_size=c.page_size, num_sms=148)
    h = hashlib.sha256()
    for k in ("header", "cta_ptr", "tiles"):
        h.update(np.ascontiguousarray(p[k]).tobytes())
    return h.hexdigest()


def _rank_main(rank, world, port, queue):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's own device time; the step time is the slowest rank's
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        digests = [None] * world
        dist.all_gather_object(digests, _plan_digest(2))
        dist.barrier()
        queue.put((rank, ms, digests))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_plan_and_time():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, ms, digests = queue.get(timeout=240)
        results[rank] = (ms, digests)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0][0] == results[1][0] == 15.0
    d0, d1 = results[0][1], results[1][1]
    assert d0 == d1 and d0[0] == d0[1], "replicas planned different work"


def test_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_gbs(1e9, 1, 2.0)
    assert one == pytest.approx(500.0)
    # weak scaling: same per-rank bytes, same slowest-rank time -> N times the job value
    assert bench.job_gbs(1e9, 4, 2.0) == pytest.approx(4 * one)
    assert bench.max_over_ranks(3.5, None) == 3.5        # outside a process group


def test_reference_arm_prints_from_rank_zero_only():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
