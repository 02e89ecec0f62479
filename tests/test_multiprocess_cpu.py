"""The N>1 host logic of bench.py on CPU: two gloo ranks, weak scaling (each rank its
own seeded sequences) and the max-over-ranks timing every rank agrees on."""
import os

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + rank, world, "cpu")
        seed = bench.rank_inputs_seed(1, rank)
        wl = synth.workload(bench.WORKLOAD)
        x = synth.layer_input(wl["cfg"], 1, 4, seed)
        out[rank] = (t, seed, float(x.sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_and_max_time():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0          # both see the slowest rank
    assert out[0][1] != out[1][1]                   # each rank draws its own inputs
    assert out[0][2] != out[1][2]
