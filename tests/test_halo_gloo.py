"""Sequence-parallel sliding window on the CPU: the halo exchange between
gloo ranks, and the shard semantics of gdla_attn_fwd_sp checked with the
float64 oracle in place of the kernel.

A sequence split across ranks: each rank receives the last HALO_ROWS K/V rows
of the previous rank's shard, and its shard's output rows, computed from
[halo | shard] alone, equal the full-sequence rows (a windowed row reads only
the W-1 keys before it)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from grouped_differential_attention_gdla_b200 import halo
from grouped_differential_attention_gdla_b200.inputs import custom, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard_rows_with_oracle(x, k_buf, v_buf, kv_prefix, start, T_loc, window):
    """Rows of one shard from the oracle over the shard's [halo | own] K/V:
    query row i reads K/V row i + kv_prefix (the kernel's shard semantics)."""
    H0 = halo.HALO_ROWS - kv_prefix
    k = k_buf[:, H0:]
    v = v_buf[:, H0:]
    loc = np.arange(T_loc, dtype=np.int64)
    sl = lambda t: t[0, start:start + T_loc]
    return oracle.gdla_attn_rows(sl(x["q_sig"]), sl(x["q_noise"]), k, v, sl(x["lam"]),
                                 sl(x["gate"]), loc + kv_prefix, window=window, causal=True)


def _worker(rank, world, port, T, window, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = custom(1, T, 8, 2, 2, 64, window=window)
        x = make_inputs(wl, seed=11)  # every rank draws the same sequence
        T_loc = T // world
        start = rank * T_loc
        k_buf = halo.kv_shard_buffer(1, T_loc, wl.Hkv, wl.d, "cpu")
        v_buf = halo.kv_shard_buffer(1, T_loc, wl.Hkv, wl.d, "cpu")
        k_buf.fill_(float("nan"))
        v_buf.fill_(float("nan"))
        k_buf[:, halo.HALO_ROWS:] = x["k"][:, start:start + T_loc]
        v_buf[:, halo.HALO_ROWS:] = x["v"][:, start:start + T_loc]
        kv_prefix = halo.exchange_halo(k_buf, v_buf)
        got_halo = None
        if rank > 0:
            got_halo = bool(torch.equal(k_buf[:, :halo.HALO_ROWS],
                                        x["k"][:, start - halo.HALO_ROWS:start]) and
                            torch.equal(v_buf[:, :halo.HALO_ROWS],
                                        x["v"][:, start - halo.HALO_ROWS:start]))
        mine = _shard_rows_with_oracle(x, k_buf, v_buf, kv_prefix, start, T_loc, window)
        full = oracle.gdla_attn_rows(x["q_sig"][0, start:start + T_loc],
                                     x["q_noise"][0, start:start + T_loc], x["k"], x["v"],
                                     x["lam"][0, start:start + T_loc],
                                     x["gate"][0, start:start + T_loc],
                                     np.arange(start, start + T_loc), window=window, causal=True)
        results[rank] = (kv_prefix, got_halo, float(np.abs(mine - full).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,window", [(3, 768, 128), (2, 512, 64), (4, 1024, 1)])
def test_halo_exchange_and_shard_rows(world, T, window):
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), T, window, results), nprocs=world, join=True)
    for r in range(world):
        kv_prefix, got_halo, err = results[r]
        assert kv_prefix == (0 if r == 0 else halo.HALO_ROWS)
        assert got_halo in (None, True)
        assert err == 0.0, f"rank {r}: shard rows differ from the full sequence by {err}"


def test_window_locality_pin():
    """Oracle invariant behind the halo: with window W a row's output depends
    only on K/V rows (i-W, i], so evaluating it on a K/V slice that starts at
    any row s <= i-W+1 (rows re-indexed by -s) gives the same value exactly."""
    wl = custom(2, 600, 8, 2, 2, 64, window=100)
    x = make_inputs(wl, seed=3)
    rows = np.array([99, 100, 250, 599, 600 + 99, 600 + 420])  # flat b*T + i
    full = oracle.gdla_attn_rows(*(t.reshape(2 * 600, *t.shape[2:])[rows] for t in
                                   (x["q_sig"], x["q_noise"])), x["k"], x["v"],
                                 x["lam"].reshape(1200, -1)[rows],
                                 x["gate"].reshape(1200, -1)[rows], rows, window=100)
    for j, flat in enumerate(rows):
        b, i = divmod(int(flat), 600)
        s = max(0, i - 99 - 7)  # any start at or before the window's first key
        k = x["k"][b:b + 1, s:i + 1]
        v = x["v"][b:b + 1, s:i + 1]
        one = oracle.gdla_attn_rows(x["q_sig"][b, i:i + 1], x["q_noise"][b, i:i + 1], k, v,
                                    x["lam"][b, i:i + 1], x["gate"][b, i:i + 1],
                                    np.array([i - s]), window=100)
        assert np.array_equal(one[0], full[j])
    # and it does depend on the key just inside the window
    k2 = x["k"].clone()
    k2[0, 250 - 99] += 1.0
    moved = oracle.gdla_attn_rows(x["q_sig"][0, 250:251], x["q_noise"][0, 250:251], k2, x["v"],
                                  x["lam"][0, 250:251], x["gate"][0, 250:251], np.array([250]),
                                  window=100)
    assert not np.array_equal(moved[0], full[2])


def test_shard_needs_a_full_halo():
    k = halo.kv_shard_buffer(1, 64, 2, 64, "cpu")
    with pytest.raises(ValueError):
        halo.exchange_halo(k, k.clone())
