"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

The path is data-parallel with no collective on the data: each rank quantizes
and multiplies its own token batch, and the only communication is the
max-over-ranks reduction of the timings. These tests run that logic in two
processes with the gloo backend (no GPU): per-rank batches, the max over
ranks, the whole-job throughput, and the reference arm's rank behaviour.
"""

import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
mp = pytest.importorskip("torch.multiprocessing")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench
    import workloads as WL
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = WL.svdq_inputs(WL.custom_svdq("mr", 96, 128, 64, 16, seed=5))["X"]
        mine = bench.rank_rows(x, rank)
        # rank-dependent step times; every rank must see the same maxima
        times = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        mx = bench.max_over_ranks(times, world, "cpu")
        val = bench.job_tflops(1e12, world, mx[0])
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), rows=mine, mx=np.array(mx),
                 val=np.array(val))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npz")
    r1 = np.load(tmp_path / "rank1.npz")
    # the same maxima on both ranks: max(1, 2), max(5, 4), max(0.25, 0.5)
    assert r0["mx"].tolist() == r1["mx"].tolist() == [2.0, 5.0, 0.5]
    # whole-job value: both ranks' work over the slowest rank's step time
    assert float(r0["val"]) == pytest.approx(1e12 * 2 / 2e-3 / 1e12)
    # weak scaling: same shape, different rows, and a permutation of the same draw
    a, b = r0["rows"], r1["rows"]
    assert a.shape == b.shape and not np.array_equal(a, b)
    assert np.array_equal(np.roll(a, 37, axis=0), b)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    args = argparse.Namespace(gpus=2, steps=1, warmup=3, cpu_budget=0)
    bench.run_reference(args, rank=1)  # a non-zero rank exits without work or output
    assert capsys.readouterr().out == ""
