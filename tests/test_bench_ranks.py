"""Host logic of bench.py's multi-GPU path on CPU (two gloo ranks).

The layer does not shard: `bench.py --gpus N` runs N independent replicas,
reports the slowest rank's time and all ranks' bytes.  These tests check that
reduction with a real two-process group (gloo on 127.0.0.1) and that the
reference arm under torch.distributed.run prints one line from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}",
                                         rank=rank, world_size=world)
    try:
        ms = [3.0, 5.5][rank]
        m = bench.max_over_ranks(ms, torch.device("cpu"))
        v = bench.whole_job_value(world, 1e9, 10, m)
        q.put((rank, m, v))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 5.5                                  # slowest rank's time on every rank
        assert v == pytest.approx(2 * 1e9 * 10 / 5.5e-3 / 1e9)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(4.25, torch.device("cpu")) == 4.25
    assert bench.whole_job_value(1, 2e9, 5, 10.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="4")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=900, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                               # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
