"""GPU parity of the GDLA attention backward against the float64 oracle.

gdla_attn_bwd (through the C ABI) returns the gradients of the forward for an
upstream gradient dO: dQ_sig, dQ_noise, dK, dV, dlambda, dG.  The oracle
(oracle.gdla_attn_bwd, pinned by finite differences and torch autograd)
computes them in float64 from the same seeded bf16 inputs.  Every element of
every gradient is compared, per tensor, with the forward's tolerance
max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3.
"""
import numpy as np
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
import oracle
from grouped_differential_attention_gdla_b200.inputs import custom, make_inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu

NAMES = ("dq_sig", "dq_noise", "dk", "dv", "dlam", "dgate")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdla.load_library()


def _case(B, T, Hs, Hn, Hkv, d, window, causal, seed):
    wl = custom(B, T, Hs, Hn, Hkv, d, window=window, causal=causal)
    x = make_inputs(wl, seed=seed, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    dout = torch.randn(B, T, Hs * d, generator=g, device="cuda").to(torch.bfloat16)
    return x, dout


def _check(x, dout, window, causal, what):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = gdla.gdla_attn_bwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], dout,
                             window=window, causal=causal, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    cpu = {k: v.cpu() for k, v in x.items()}
    ref = oracle.gdla_attn_bwd(cpu["q_sig"], cpu["q_noise"], cpu["k"], cpu["v"], cpu["lam"],
                               cpu["gate"], dout.cpu(), window=window, causal=causal)
    for n in NAMES:
        assert_parity(got[n].float().cpu().numpy(), ref[n], f"bwd {n} {what}")


EDGE = [
    # B, T, Hs, Hn, Hkv, d, window, causal
    (1, 256, 8, 2, 2, 64, 0, True),      # the tiny shape
    (1, 1, 8, 2, 2, 128, 0, True),       # one token
    (2, 127, 8, 2, 2, 128, 0, True),     # ragged single tile
    (1, 129, 8, 2, 2, 128, 0, True),     # one row into a second tile
    (1, 300, 4, 4, 4, 128, 0, True),     # g = 1
    (1, 300, 6, 2, 2, 64, 0, True),      # g = 3
    (1, 700, 8, 2, 2, 128, 1, True),     # window of one key
    (1, 700, 8, 2, 2, 128, 128, True),   # the Motif 3 window
    (1, 700, 8, 2, 2, 64, 200, True),    # window wider than a tile
    (1, 333, 8, 2, 2, 128, 0, False),    # no mask
    (2, 600, 8, 2, 2, 128, 0, True),
]


@pytest.mark.parametrize("B,T,Hs,Hn,Hkv,d,window,causal", EDGE)
def test_bwd_every_element(B, T, Hs, Hn, Hkv, d, window, causal):
    x, dout = _case(B, T, Hs, Hn, Hkv, d, window, causal, seed=T + window + d)
    _check(x, dout, window, causal, f"{B},{T},{Hs},{Hn},{d},{window},{causal}")


@pytest.mark.parametrize("window", [0, 128])
def test_bwd_motif_heads(window):
    """The Motif 3 head counts (64 signal / 16 noise / 16 KV heads, d = 128)
    over 1024 tokens, full causal and the 128-token window."""
    x, dout = _case(1, 1024, 64, 16, 16, 128, window, True, seed=31 + window)
    _check(x, dout, window, True, f"64/16/16 T=1024 W={window}")


def test_bwd_deterministic():
    x, dout = _case(1, 500, 8, 2, 2, 128, 0, True, seed=3)
    a = gdla.gdla_attn_bwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], dout)
    b = gdla.gdla_attn_bwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], dout)
    torch.cuda.synchronize()
    gdla.check_status()
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n
