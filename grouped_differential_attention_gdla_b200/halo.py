"""Sequence-parallel sliding-window GDLA: one halo exchange between ranks.

A sequence of T tokens is split across P ranks, rank r holding the shard of
tokens [r*T_loc, (r+1)*T_loc).  In a sliding-window layer (W <= 128) a query
token reads only the W-1 keys before it, so a rank needs just the last keys
of the previous rank's shard, the halo: one point-to-point exchange per layer
in place of the P-1 K/V rotations of ring attention ("Motif 3: Technical
Report", paper.rainbus.top, long-context training step and "technical
novelty" paragraph: window-aware ring attention for the sliding layers, a
single halo exchange that cuts each rank's K/V receive from Theta(L) to
Theta(W)).

Each rank keeps its K and V shards in buffers with HALO_ROWS rows of
headroom in front (kv_shard_buffer).  exchange_halo() sends the shard's last
HALO_ROWS rows to the next rank and receives the previous rank's into the
headroom; gdla_attn_fwd_sequence_parallel() then runs the shard through the
library's gdla_attn_fwd_sp.  The exchange uses torch.distributed
point-to-point calls (NCCL between GPUs, gloo between CPU processes); every
rank must call it in the same order.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import _binding

HALO_ROWS = 128  # one K/V tile: covers any window of up to 128 keys
MAX_WINDOW = 128


def kv_shard_buffer(B: int, T_loc: int, Hkv: int, d: int, device,
                    dtype=torch.bfloat16) -> torch.Tensor:
    """A [B, HALO_ROWS + T_loc, Hkv, d] buffer for one K (or V) shard: the
    shard's own rows go to [:, HALO_ROWS:], the exchange fills [:, :HALO_ROWS]."""
    return torch.empty((B, HALO_ROWS + T_loc, Hkv, d), dtype=dtype, device=device)


def _peers(group) -> Tuple[int, int, Optional[int], Optional[int]]:
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    glob = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    prev = glob(rank - 1) if rank > 0 else None
    nxt = glob(rank + 1) if rank + 1 < world else None
    return rank, world, prev, nxt


def exchange_halo(k_buf: torch.Tensor, v_buf: torch.Tensor, group=None) -> int:
    """Send this rank's last HALO_ROWS K/V rows to the next rank and receive
    the previous rank's into the headroom of k_buf / v_buf.

    Returns the kv_prefix for gdla_attn_fwd_sp: HALO_ROWS, or 0 on the first
    rank (no keys precede its shard; its headroom is left untouched).
    """
    if k_buf.shape != v_buf.shape or k_buf.dim() != 4:
        raise ValueError("k_buf and v_buf must be [B, HALO_ROWS + T_loc, Hkv, d] alike")
    T_loc = k_buf.shape[1] - HALO_ROWS
    if T_loc < HALO_ROWS:
        raise ValueError(f"a shard must hold at least {HALO_ROWS} tokens, got {T_loc}")
    rank, world, prev, nxt = _peers(group)
    reqs = []
    recv = None
    if nxt is not None:
        for buf in (k_buf, v_buf):
            reqs.append(dist.isend(buf[:, -HALO_ROWS:].contiguous(), dst=nxt, group=group))
    if prev is not None:
        recv = [torch.empty_like(k_buf[:, :HALO_ROWS]) for _ in range(2)]
        for t in recv:
            reqs.append(dist.irecv(t, src=prev, group=group))
    for r in reqs:
        r.wait()
    if recv is None:
        return 0
    k_buf[:, :HALO_ROWS].copy_(recv[0])
    v_buf[:, :HALO_ROWS].copy_(recv[1])
    return HALO_ROWS


def gdla_attn_fwd_sequence_parallel(q_sig, q_noise, k_buf, v_buf, lam, gate, window: int,
                                    group=None, scale: float = 0.0, out=None, d_status=None,
                                    stream=None) -> torch.Tensor:
    """Sliding-window GDLA forward of this rank's shard of a sequence.

    q_sig [B,T_loc,Hs,d], q_noise [B,T_loc,Hn,d], lam [B,T_loc,Hs] and gate
    [B,T_loc,Hs*d] hold the shard's tokens; k_buf / v_buf are kv_shard_buffer
    tensors with the shard's K / V in [:, HALO_ROWS:].  Exchanges the halo,
    then computes out [B, T_loc, Hs*d].  window in 1..128.
    """
    if not 0 < window <= MAX_WINDOW:
        raise ValueError(f"window must be in 1..{MAX_WINDOW} for the halo exchange")
    kv_prefix = exchange_halo(k_buf, v_buf, group)
    B, T_loc = q_sig.shape[0], q_sig.shape[1]
    if out is None:
        out = torch.empty((B, T_loc, q_sig.shape[2] * q_sig.shape[3]), dtype=torch.bfloat16,
                          device=q_sig.device)
    if kv_prefix or B == 1:
        k = k_buf[:, HALO_ROWS - kv_prefix:]
        v = v_buf[:, HALO_ROWS - kv_prefix:]
        return _binding.gdla_attn_fwd_sp(q_sig, q_noise, k, v, lam, gate, window, kv_prefix,
                                         scale=scale, out=out, d_status=d_status, stream=stream)
    # first rank with several sequences: [:, HALO_ROWS:] is strided across the
    # batch, so each sequence runs on its own contiguous view
    for b in range(B):
        _binding.gdla_attn_fwd_sp(q_sig[b:b + 1], q_noise[b:b + 1], k_buf[b:b + 1, HALO_ROWS:],
                                  v_buf[b:b + 1, HALO_ROWS:], lam[b:b + 1], gate[b:b + 1],
                                  window, 0, scale=scale, out=out[b:b + 1], d_status=d_status,
                                  stream=stream)
    return out
