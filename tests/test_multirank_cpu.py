"""The N > 1 host path on CPU: world_size-2 `gloo` ranks (no GPU).

Rows of the linear are independent (sglang PR "Tune Kitchen INT8 row
splitting for SM120", Accuracy Test: split and single-call outputs are
bit-exact), so the benchmark either runs one replica per rank or splits the
batch's rows over the ranks, with no collective on the data path; timings are
reduced with a max over ranks. These tests run that host logic with the CPU
oracle standing in for the per-rank kernels.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("M,world", [(1, 1), (7, 2), (8, 2), (37, 3), (32700, 8), (5, 8)])
def test_shard_rows_partition(M, world):
    spans = [bench.shard_rows(M, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == M
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def _rank_main(rank, world, port, result_dir):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        import workloads

        cfg = workloads.custom(37, 512, 40, seed=5)
        X, W, bias = workloads.make_inputs(cfg)
        Qw, s_w = oracle.rotate_quant_weight(W.numpy())
        bb = workloads.bf16_bits(bias)
        lo, hi = bench.shard_rows(cfg.M, rank, world)
        Y_part = oracle.int8_linear(workloads.bf16_bits(X[lo:hi]), Qw, s_w, bb)[0]
        parts = [None] * world
        dist.all_gather_object(parts, (lo, hi, Y_part))
        # the slowest rank's time is the job's time
        mx = bench.max_over_ranks([float(rank + 1), float(-rank)])
        if rank == 0:
            parts.sort(key=lambda p: p[0])
            Y = np.concatenate([p[2] for p in parts])
            Y_full = oracle.int8_linear(workloads.bf16_bits(X), Qw, s_w, bb)[0]
            ok = np.array_equal(Y, Y_full) and mx == [float(world), 0.0]
            with open(os.path.join(result_dir, "ok" if ok else "mismatch"), "w") as f:
                f.write(repr(mx))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_rows_and_reduce_timings(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    assert (tmp_path / "ok").exists(), os.listdir(tmp_path)


def test_bench_starts_its_own_ranks():
    """`bench.py --gpus 2` launches two ranks itself (torch.distributed.run on
    127.0.0.1); the dry run does the rank plumbing on gloo with no GPU work and
    rank 0 alone prints one JSON line reporting both GPUs."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--dry-run", "--steps", "3", "--warmup", "3"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["dry_run"] and line["ms_per_step"] > 0
    assert line["config"]["parallelism"].startswith("replicas x2")
