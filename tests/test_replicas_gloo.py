"""The multi-GPU path of bench.py is independent replicas: no data-path
collective, one barrier-bracketed timing, the maximum over ranks reported by
rank 0.  This runs that host logic as two gloo ranks on the CPU."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench._dist()
        assert (w, r, lr) == (world, rank, rank)
        dist.barrier()
        mine = 10.0 + 7.5 * rank          # this rank's elapsed time
        results[rank] = (bench.max_over_ranks(mine, w), bench.replica_seed(r))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_seeds_with_two_gloo_ranks():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    assert results[0][0] == results[1][0] == 17.5   # every rank sees the slowest time
    assert {results[0][1], results[1][1]} == {0, 1}  # replicas draw different inputs


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
