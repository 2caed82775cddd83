"""The multi-rank plumbing of bench.py, on CPU with the gloo backend.

Decode sequences are independent, so N ranks each run their own batch and
exchange nothing on the data path; the only collectives are the barriers and
the max-over-ranks of the timed region.  These tests run world_size-2 process
groups on the host: the max reduction, the whole-job throughput, distinct
per-rank inputs, and the reference arm under torchrun (rank 0 prints one
line, the other rank exits 0 without work).
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    from sparse_attention_pool_b200 import configs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        dist.barrier()
        # each rank's timed region differs; all must end up with the slowest
        total = bench.max_over_ranks(10.0 + 5.0 * rank, world, dev)
        e2e = bench.max_over_ranks(30.0 - rank, world, dev)
        w = configs.BY_NAME["decode_b1_t4k_h8_k64"]
        lengths, K, V, KI, q, qI = bench.make_inputs(w, rank)
        digest = float(np.asarray(K[0, :64]).view(np.uint16).astype(np.float64).sum())
        got = torch.tensor([digest], dtype=torch.float64)
        allv = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allv, got)
        dist.barrier()
        out.put((rank, total, e2e, [float(x.item()) for x in allv],
                 bench.job_throughput(w.B * 20, world, total)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_run_distinct_sequences():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, total, e2e, digests, thr in res:
        assert total == 15.0          # the slowest rank's time, on every rank
        assert e2e == 30.0
        assert digests[0] != digests[1]  # each rank drew its own sequences
        # whole-job throughput: both ranks' 20 steps x 1 sequence over 15 ms
        assert thr == pytest.approx(2 * 20 / 0.015)


def test_single_rank_max_is_identity_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(12.5, 1, torch.device("cpu")) == 12.5
    assert bench.job_throughput(4 * 10, 1, 1000.0) == pytest.approx(40.0)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           "bench.py", "--impl", "reference", "--gpus", "2", "--workload", "decode_b1_t4k_h8_k64",
           "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["unit"] == d["unit"]
