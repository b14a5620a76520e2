"""Host logic of the multi-process benchmark on CPU: two ranks over the gloo backend
(loopback rendezvous), no GPU.  The data path has no collective; the ranks only agree on
the slowest rank's time, and the reference arm prints from rank 0 alone."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, loc = bench.rank_env()
        local_ms = 10.0 + 7.5 * rank          # rank 1 is the slowest
        ms = bench.max_over_ranks(local_ms, dist, device="cpu")
        rate = bench.whole_job_rate(w, 100, ms)
        out.put((r, w, loc, ms, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ranks_agree_on_the_slowest_time_and_the_whole_job_rate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == world and r[2] == r[0] for r in res)
    for (_, _, _, ms, rate) in res:
        assert ms == 17.5                          # the max over ranks, the same on every rank
        assert rate == pytest.approx(world * 100 / 0.0175)   # all ranks' steps over the slowest time


def test_single_process_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_rate(1, 50, 1000.0) == pytest.approx(50.0)


def test_reference_arm_prints_one_line_from_rank_zero_under_torchrun():
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "3", "--warmup", "3", "--cpu-seconds", "0.3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
