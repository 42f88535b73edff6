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


def test_kernel_labels_follow_the_dispatch_rule():
    from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, custom
    assert bench.attn_kernel_name(WORKLOADS["long_window"]) == "gdla_attn_win_kernel"
    assert bench.attn_kernel_name(WORKLOADS["window"]) == "gdla_attn_win_kernel"
    assert bench.attn_kernel_name(WORKLOADS["long_full"]) == "gdla_attn_fwd_kernel"
    assert bench.attn_kernel_name(custom(1, 700, 8, 2, 2, 128, window=200)) == \
        "gdla_attn_fwd_kernel<window>"
    assert bench.attn_kernel_name(custom(1, 700, 8, 2, 2, 128, window=700)) == \
        "gdla_attn_fwd_kernel"
    assert bench.STEPS["long"] == ("long_full", "long_window")


def test_roofline_entry_picks_bound_and_peak():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    # tensor-bound: 1.6e15 FLOP, 1e9 bytes in 1 s
    e = bench._roofline_entry("x", "k", 1.6e15, 1e9, 1000.0, peaks, "measured", False, None)
    assert e["bound"] == "tensor" and e["peak"] == 1600.0 and abs(e["frac"] - 1.0) < 1e-9
    e = bench._roofline_entry("x", "k", 1.4e15, 1e9, 1000.0, peaks, "measured", True, None)
    assert e["peak"] == 1400.0 and abs(e["frac"] - 1.0) < 1e-9
    # HBM-bound: 3e12 bytes/s against 6000 GB/s
    e = bench._roofline_entry("x", "k", 1e12, 3e12, 1000.0, peaks, "measured", True, 5)
    assert e["bound"] == "hbm" and abs(e["frac"] - 0.5) < 1e-9 and e["traffic"] == 5
