"""The multi-rank host logic of bench.py on two gloo ranks (CPU, no GPU).

The path shards as replicas: every rank draws its own tokens against the
same weights, the job time is the slowest rank's, launch counts add up, and
the reported value is all ranks' work over that time (weak scaling).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from fp8_block_scaled_group_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        slow = bench.max_over_ranks(10.0 + rank, world, device="cpu")
        launches = bench.sum_over_ranks(40.0 + rank, world, device="cpu")
        seed = bench.rank_input_seed(1004, rank, 0)
        x = inputs.activations(8, 256, seed)
        bench.barrier(world)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), slow=slow, launches=launches, seed=seed, x=x)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    assert float(r[0]["slow"]) == float(r[1]["slow"]) == 11.0       # the slowest rank's time
    assert float(r[0]["launches"]) == float(r[1]["launches"]) == 81.0  # 40 + 41
    assert int(r[0]["seed"]) != int(r[1]["seed"])                   # each rank its own tokens
    assert not np.array_equal(r[0]["x"], r[1]["x"])


def test_weak_scaling_value():
    # 2 ranks x 20 steps x 1e12 flop in 100 ms of the slowest rank
    assert bench.weak_scaling_value(1e12, 2, 20, 100.0) == pytest.approx(4e14)
    assert bench.weak_scaling_value(1e12, 1, 20, 100.0) == pytest.approx(2e14)
    assert bench.max_over_ranks(3.5, 1) == 3.5 and bench.sum_over_ranks(3.5, 1) == 3.5
    assert [bench.rank_input_seed(1004, r, i) for r in range(2) for i in range(bench.N_SETS)] == \
        sorted(set(bench.rank_input_seed(1004, r, i) for r in range(2) for i in range(bench.N_SETS)))
