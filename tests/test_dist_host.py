"""Host logic of the multi-process bench on CPU: two gloo ranks over 127.0.0.1.

On the GPU the bench runs one process per GPU and each rank is an independent
replica of the layer (its own seeded tokens and weights); the process group
carries only barriers and the max over ranks of the timings.  These tests run
that logic with the gloo backend on the host: the max-over-ranks reduction,
the per-rank seeding of the replicas, the whole-job throughput and the
reference arm, which only rank 0 runs.
"""
from __future__ import annotations

import hashlib
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def digest(t: torch.Tensor) -> str:
    return hashlib.sha256(t.contiguous().view(torch.uint8).numpy().tobytes()).hexdigest()


def _rank_env(rank: int, port: int):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(WORLD),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _worker_collectives(rank: int, port: int):
    _rank_env(rank, port)
    import torch.distributed as dist

    import bench
    from bit_post_quantised_b200 import workloads

    world, r, local = bench.setup_dist("gloo")
    try:
        assert (world, r, local) == (WORLD, rank, rank)
        # each rank "measured" a different time: every rank must get the slowest
        got = bench.max_over_ranks(0.25 + rank, world)
        assert got == 0.25 + (WORLD - 1), got
        got = bench.max_over_ranks(3.0 - rank, world)
        assert got == 3.0, got
        bench.barrier(world)

        # replicas: two input sets per rank, all distinct, reproducible
        layer = workloads.CONFIGS["tiny"]
        sets = bench.make_sets(layer, rank, 2, torch.device("cpu"))
        again = bench.make_sets(layer, rank, 2, torch.device("cpu"))
        mine = []
        for a, b in zip(sets, again):
            for key in ("x", "W", "b"):
                assert digest(a[key]) == digest(b[key])
            assert a["y"].shape == (layer.M, layer.N)
            assert a["packed"].numel() == layer.N * layer.K // 4
            assert a["scales"].numel() == layer.N
            mine.append((digest(a["x"]), digest(a["W"])))
        everyone = [None] * world
        dist.all_gather_object(everyone, mine)
        flat = [h for per_rank in everyone for pair in per_rank for h in pair]
        assert len(set(flat)) == len(flat), "two replicas share inputs"

        # whole-job throughput counts every rank's steps over the slowest time
        elapsed = bench.max_over_ranks(0.5 * (rank + 1), world)
        v = bench.job_throughput(world, 10, layer.flop, elapsed)
        assert v == pytest.approx(WORLD * 10 * layer.flop / (0.5 * WORLD) / 1e12)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_seed_and_throughput():
    mp.start_processes(_worker_collectives, args=(free_port(),), nprocs=WORLD, join=True,
                       start_method="spawn")


def _worker_reference(rank: int, port: int, out_dir: str):
    _rank_env(rank, port)
    import argparse
    import contextlib
    import io

    import bench

    args = argparse.Namespace(gpus=WORLD, steps=1, warmup=0, impl="reference", workload="tiny",
                              no_extras=True, cpu_seconds=0.0)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(args)
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(f"{rc}\n{buf.getvalue()}")


def test_reference_arm_runs_on_rank0_only(tmp_path):
    """Under torchrun every rank starts the reference arm; rank 0 alone times
    the oracle and prints the line, the others exit 0 without work."""
    import json

    mp.start_processes(_worker_reference, args=(free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    rc0, out0 = (tmp_path / "rank0.txt").read_text().split("\n", 1)
    rc1, out1 = (tmp_path / "rank1.txt").read_text().split("\n", 1)
    assert rc0 == "0" and rc1 == "0"
    assert out1.strip() == ""
    lines = [ln for ln in out0.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == WORLD and line["steps"] == 1
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
