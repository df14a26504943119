"""Multi-process host logic of the replicated decode path, on CPU with gloo.

Two ranks: token sharding is disjoint and covers the stream, the timing
reduction is a maximum over ranks, and the whole-job throughput counts every
rank's tokens over the slowest rank's time.  The reference arm of bench.py,
launched under torchrun with two ranks, prints exactly one result line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from activation_sparse_ffn_predict_b200 import replicas as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sl = R.token_slice(rank, world, 5)
        mine = float(10 + 7 * rank)              # ranks take different times
        mx = R.max_over_ranks(mine)
        R.barrier()
        q.put((rank, sl.start, sl.stop, mx, R.job_throughput(5, world, mx)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [(r[1], r[2]) for r in res] == [(0, 5), (5, 10)]
    assert all(r[3] == 17.0 for r in res)                 # max over ranks
    assert all(abs(r[4] - 10 / 0.017) < 1e-6 for r in res)  # 10 tokens in 17 ms


def test_single_process_helpers():
    assert R.max_over_ranks(3.5) == 3.5
    assert R.token_slice(1, 4, 8) == slice(8, 16)
    with pytest.raises(ValueError):
        R.token_slice(4, 4, 8)
    with pytest.raises(ValueError):
        R.job_throughput(1, 1, 0.0)


def test_reference_arm_under_torchrun_prints_one_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "3",
           "--warmup", "1", "--config", "tiny_reglu_f32", "--reference-budget", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
