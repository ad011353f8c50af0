"""The multi-rank host logic of bench.py on CPU: two gloo ranks (world_size 2).

Each rank runs its own batch (weak scaling, no collective on the data path); the timings
are combined as the max over ranks and the throughput counts the units of all ranks.
"""
import importlib.util
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("kda_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = load_bench()
        # rank r pretends its timed region took (1 + r) ms per step
        per_rank = [10.0 * (1 + rank), 7.0 + rank, 3.0 - rank]
        combined = bench.max_over_ranks(per_rank, "cpu", world)
        tput = bench.weak_scaling_throughput(32768, world, 10, combined[1] / 1e3)
        out[rank] = (combined, tput)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_two_gloo_ranks():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = 29500 + (os.getpid() % 1000)
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for r in range(2):
        combined, tput = out[r]
        assert combined == [20.0, 8.0, 3.0]             # element-wise max over the two ranks
        assert tput == pytest.approx(2 * 32768 * 10 / 8e-3)


def test_single_rank_is_identity():
    bench = load_bench()
    assert bench.max_over_ranks([1.5, 2.5], "cpu", 1) == [1.5, 2.5]
    assert bench.weak_scaling_throughput(100, 1, 4, 2.0) == 200.0
