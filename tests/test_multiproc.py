"""The N > 1 plumbing of bench.py on CPU: gloo ranks, world size 2.

The path shards into independent (sequence, head) units, so N GPUs run N
replicas with no data-path collective; the only cross-rank steps are the
barrier and the max-over-ranks reduction of the measured time.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank          # the slower rank sets the time
        t = bench.max_over_ranks(local_ms, ws)
        rate = bench.whole_job_rate(16384, ws, t / 1e3)
        q.put((rank, t, rate, bench.rank_seeds(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(ws))
    for rank, t, rate, seeds in res:
        assert t == 15.0                       # max over ranks
        assert rate == pytest.approx(2 * 16384 / 0.015)
    assert set(res[0][3]).isdisjoint(res[1][3])  # each replica draws its own batch


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                    # rank 0 alone prints
    obj = json.loads(lines[0])
    assert obj["impl"] == "reference" and obj["unit"] == "tokens/s" and obj["value"] > 0
    assert obj["e2e"]["h2d_bytes_per_step"] == 0
