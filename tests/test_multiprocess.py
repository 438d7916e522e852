"""The N > 1 path on CPU: world_size-2 `gloo` process groups and a two-rank
torchrun launch of the benchmark's reference arm.

The method's (b, h) problems are independent, so `bench.py --gpus N` runs one
replica of the workload per GPU with no data-path collective; the only
exchange is the timing: the job's time is the slowest rank's (max over ranks)
and its throughput counts every rank's tokens. These tests cover that host
logic without a GPU.
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

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        times = [12.5, 20.0]  # ms: rank 1 is the slower one
        mx = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        value = bench.job_tokens_per_s(1000, world, 10, mx)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "value": value}, f)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        got = json.load(open(tmp_path / f"rank{r}.json"))
        assert got["max"] == 20.0
        # every rank's 10 x 1000 tokens over the slowest rank's 20 ms
        assert got["value"] == pytest.approx(2 * 10 * 1000 / 0.020)


def test_without_a_process_group_the_time_is_the_rank_own():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--config", "c1", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 2


def test_attention_flop_count_matches_a_brute_force_count():
    """bench.attn_flops against 4 D times the visible (query token, key
    token) pairs counted one by one, causal and not, with grouped queries and
    -1 padded lists."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench

    rng = np.random.default_rng(3)
    B, H, Hk, nb, bs, D, kk = 2, 4, 2, 6, 8, 16, 3
    N = nb * bs
    idx = np.full((B, Hk, nb, kk), -1, np.int64)
    for b in range(B):
        for g in range(Hk):
            for i in range(nb):
                n = min(kk, i + 1)
                idx[b, g, i, :n] = np.sort(rng.choice(i + 1, n, replace=False))
    brute = 0
    for b in range(B):
        for g in range(Hk):
            for i in range(nb):
                for j in idx[b, g, i]:
                    if j < 0:
                        continue
                    for r in range(bs):
                        for c in range(bs):
                            brute += (j * bs + c) <= (i * bs + r)
    assert bench.attn_flops(B, H, Hk, N, D, bs, kk, idx, causal=True) == 4.0 * D * brute * (H // Hk)
    full = B * H * N * kk * bs  # every query token sees k * bs keys
    assert bench.attn_flops(B, H, Hk, N, D, bs, kk) == 4.0 * D * full
