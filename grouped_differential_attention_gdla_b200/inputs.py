"""Seeded synthetic inputs for the GDLA forward pass.

This module is the one piece shared by the CUDA path's tests and benchmark and
by the float64 oracle's tests: it only draws random numbers and lays them out.
It holds none of the method's arithmetic (the sigmoid below prepares the
already-activated lambda and gate inputs, which arrive at the attention
boundary as given values).

Recipe (fixed order, one ``torch.Generator`` seeded once; decode workloads
draw Q_sig, Q_noise [B, H, d], lambda, gate, the cache's raw latents
c_KV [B, T, 512] and W^KV_b in that order):
  Q_sig, Q_noise, K, V  ~ N(0, 1) rounded to bfloat16   (K, V skipped for the
                                                           latent workload)
  lambda = bf16(sigmoid(N(0, 1)))  shape [B, T, Hs]
  gate   = bf16(sigmoid(N(0, 1)))  shape [B, T, Hs*d]
  c_KV   ~ N(0, 1) bf16            shape [B*T, 512]      (latent workload)
  W^KV_b ~ N(0, 1/512) bf16        shape [512, Hkv*(dk+dv)]
then, for backward workloads, the upstream gradient dO ~ N(0, 1) bf16
[B, T, Hs*d]; and, for workloads with the decoupled rotary term (d_rope > 0),
drawn after everything above so the other inputs do not change:
  Q_rope_sig, Q_rope_noise ~ N(0, 1) bf16  shape [B, T, H, d_rope]
  K_rope                   ~ N(0, 1) bf16  shape [B, T, d_rope]
The same seed on a different device gives a different (but again fixed)
stream; tests that compare against the oracle copy the device draw to the host.

Workload shapes follow the pages' Motif 3 attention: 64 signal / 16 noise
query heads over 16 shared KV heads, head dim 128, sliding window 128 or full
causal ("Вышла новая модель Motif 3", pikabu.ru; "Motif 3: Technical Report",
paper.rainbus.top, step 2).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hs: int = 64
    Hn: int = 16
    Hkv: int = 16
    d: int = 128
    window: int = 0          # 0 = full causal; W > 0 keeps keys i-W < j <= i
    causal: bool = True
    latent: bool = False     # K, V come from RMSNorm + W^KV_b of c_KV
    d_latent: int = 512
    eps: float = 1e-6
    decode: bool = False     # one query token per sequence over a T-token latent cache
    d_rope: int = 0          # width of the decoupled rotary term (0: none)
    bwd: bool = False        # the backward: gradients for an upstream dO

    @property
    def g(self) -> int:
        return self.Hs // self.Hn

    def pairs_per_batch(self) -> int:
        """(query, key) pairs the mask keeps in one batch element."""
        T, W = self.T, self.window
        if self.decode:  # the newest token over a full cache of T tokens
            return min(T, W) if W > 0 else T
        if not self.causal:
            return T * T
        if W <= 0 or W >= T:
            return T * (T + 1) // 2
        # rows i < W keep i+1 keys, the rest keep W
        return W * (W + 1) // 2 + (T - W) * W

    def attn_flops(self) -> int:
        """2*(d + d_rope) + 2*d FLOPs per kept pair per query head (QK^T with
        the rotary term, and PV), all heads."""
        per_pair = 2 * (self.d + self.d_rope) + 2 * self.d
        return per_pair * (self.Hs + self.Hn) * self.B * self.pairs_per_batch()

    def decode_bytes(self) -> int:
        """The kept cache rows read once, W^KV_b, the query-side inputs and
        the output, bfloat16 everywhere."""
        per_seq = self.pairs_per_batch() * self.d_latent + (self.Hs + self.Hn) * self.d + \
            self.Hs + 2 * self.Hs * self.d
        return 2 * (self.B * per_seq + self.d_latent * self.Hkv * 2 * self.d)

    def attn_bytes(self) -> int:
        """Inputs read once plus output written once, bfloat16 everywhere."""
        per_tok = 2 * (self.Hs * self.d + self.Hn * self.d + 2 * self.Hkv * self.d
                       + self.Hs + 2 * self.Hs * self.d
                       + (self.Hs + self.Hn + 1) * self.d_rope)
        return per_tok * self.B * self.T

    def bwd_flops(self) -> int:
        """The backward's algorithmic work: S recomputed, dP, dS K, dS^T Q and
        P^T dO, 2*d FLOPs each per kept pair per head (10*d, 2.5x the
        forward's 4*d)."""
        return 10 * self.d * (self.Hs + self.Hn) * self.B * self.pairs_per_batch()

    def bwd_bytes(self) -> int:
        """The forward's inputs and dO read once, the six gradients written
        once, bfloat16 everywhere."""
        per_tok = 2 * (2 * (self.Hs * self.d + self.Hn * self.d + 2 * self.Hkv * self.d
                            + self.Hs + self.Hs * self.d) + self.Hs * self.d)
        return per_tok * self.B * self.T

    def expand_flops(self) -> int:
        return 2 * self.B * self.T * self.d_latent * self.Hkv * 2 * self.d

    def expand_bytes(self) -> int:
        n = self.B * self.T
        return 2 * (n * self.d_latent + self.d_latent * self.Hkv * 2 * self.d
                    + n * self.Hkv * 2 * self.d)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, T=256, Hs=8, Hn=2, Hkv=2, d=64),
    "window": Workload("window", B=8, T=4096, window=128),
    "full": Workload("full", B=2, T=8192),
    "latent": Workload("latent", B=1, T=32768, latent=True),
    "long_full": Workload("long_full", B=1, T=131072),
    "long_window": Workload("long_window", B=1, T=262144, window=128),
    # decode: 64 sequences, each with a 32768-token latent cache (the 32K stage
    # of the long-context schedule), every key or the 128-token window
    "decode": Workload("decode", B=64, T=32768, decode=True),
    "decode_window": Workload("decode_window", B=64, T=32768, window=128, decode=True),
    # the two attention layers with the decoupled rotary term (64 wide, the
    # width that keeps the latent cache the size of MLA's: 512 + 64)
    "full_rope": Workload("full_rope", B=2, T=8192, d_rope=64),
    "window_rope": Workload("window_rope", B=8, T=4096, window=128, d_rope=64),
    # the backward of the full-attention and sliding-window layers
    "bwd_full": Workload("bwd_full", B=2, T=8192, bwd=True),
    "bwd_window": Workload("bwd_window", B=8, T=4096, window=128, bwd=True),
}


def _normal_bf16(shape, gen, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def _sigmoid_bf16(shape, gen, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return torch.sigmoid_(x).to(torch.bfloat16)


def make_inputs(wl: Workload, seed: int = 0, device="cpu",
                T: Optional[int] = None, B: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw every input of one workload (optionally with B or T overridden).

    Returns a dict with q_sig [B,T,Hs,d], q_noise [B,T,Hn,d], lam [B,T,Hs],
    gate [B,T,Hs*d] and either k, v [B,T,Hkv,d] or, for the latent workload,
    c_kv [B*T, d_latent] and w_kvb [d_latent, Hkv*2d].
    """
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {}
    if wl.decode:
        # one query token per sequence; the cache holds raw KV latents
        out["q_sig"] = _normal_bf16((B, wl.Hs, wl.d), gen, device)
        out["q_noise"] = _normal_bf16((B, wl.Hn, wl.d), gen, device)
        out["lam"] = _sigmoid_bf16((B, wl.Hs), gen, device)
        out["gate"] = _sigmoid_bf16((B, wl.Hs * wl.d), gen, device)
        out["c_kv"] = _normal_bf16((B, T, wl.d_latent), gen, device)
        out["w_kvb"] = _normal_bf16((wl.d_latent, wl.Hkv * 2 * wl.d), gen, device,
                                    std=(1.0 / wl.d_latent) ** 0.5)
        return out
    out["q_sig"] = _normal_bf16((B, T, wl.Hs, wl.d), gen, device)
    out["q_noise"] = _normal_bf16((B, T, wl.Hn, wl.d), gen, device)
    if not wl.latent:
        out["k"] = _normal_bf16((B, T, wl.Hkv, wl.d), gen, device)
        out["v"] = _normal_bf16((B, T, wl.Hkv, wl.d), gen, device)
    out["lam"] = _sigmoid_bf16((B, T, wl.Hs), gen, device)
    out["gate"] = _sigmoid_bf16((B, T, wl.Hs * wl.d), gen, device)
    if wl.latent:
        out["c_kv"] = _normal_bf16((B * T, wl.d_latent), gen, device)
        out["w_kvb"] = _normal_bf16((wl.d_latent, wl.Hkv * 2 * wl.d), gen, device,
                                    std=(1.0 / wl.d_latent) ** 0.5)
    if wl.bwd:
        out["d_out"] = _normal_bf16((B, T, wl.Hs * wl.d), gen, device)
    if wl.d_rope:
        out["q_rope_sig"] = _normal_bf16((B, T, wl.Hs, wl.d_rope), gen, device)
        out["q_rope_noise"] = _normal_bf16((B, T, wl.Hn, wl.d_rope), gen, device)
        out["k_rope"] = _normal_bf16((B, T, wl.d_rope), gen, device)
    return out


def custom(B: int, T: int, Hs: int, Hn: int, Hkv: int, d: int, window: int = 0,
           causal: bool = True, latent: bool = False, name: str = "custom",
           d_rope: int = 0) -> Workload:
    """A workload with arbitrary shapes (edge-case tests)."""
    return Workload(name, B=B, T=T, Hs=Hs, Hn=Hn, Hkv=Hkv, d=d, window=window,
                    causal=causal, latent=latent, d_rope=d_rope)
