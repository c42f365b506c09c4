"""Multi-rank plumbing of bench.py on CPU with gloo (world size 2).

The path partitions into independent batches, one per GPU, so the only
collective is the max-over-ranks of the timed region."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from segmented_kv_cache_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        wl = synth.make_workload(4, values=False, seed=bench.rank_seed(4, rank))
        lens = torch.tensor(wl.batches[0].k_lens, dtype=torch.float64)
        gathered = [torch.zeros_like(lens) for _ in range(world)]
        dist.all_gather(gathered, lens)
        out[rank] = (slowest, bench.job_throughput(world, 100.0, slowest, 4),
                     bool(torch.equal(gathered[0], gathered[1])), wl.num_slots > 0)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_draw_distinct_batches():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        slowest, rate, same_lengths, ok = out[rank]
        assert slowest == 15.0                       # max over ranks, on every rank
        assert rate == pytest.approx(2 * 100.0 / (15e-3 / 4))
        assert not same_lengths                      # each rank has its own batch
        assert ok


def test_single_process_helpers():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_seed(5, 0) == 4 and bench.rank_seed(5, 1) == 1004
    assert bench.job_throughput(1, 50.0, 10.0, 2) == pytest.approx(50.0 / 5e-3)
