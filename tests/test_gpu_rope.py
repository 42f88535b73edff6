"""GPU parity of the GDLA attention forward with the decoupled rotary term.

The score adds q_r . k_r, with one rotary key per token shared by every head
of both query paths ("Motif 3: Technical Report", paper.rainbus.top, its
"technical novelty" paragraph).  Every call goes through the C ABI
(gdla_attn_fwd_rope); the reference is the float64 oracle on the same seeded
bf16 inputs.  Small shapes are compared on every element, the full-size
workloads on sampled rows (an output row depends only on its own query row and
the keys its mask keeps, so the oracle evaluates those rows alone).
Tolerance (per tensor): max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3.
"""
import numpy as np
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
import oracle
from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, custom, make_inputs
from parity import assert_parity, gather_rows, sample_rows

pytestmark = pytest.mark.gpu

ROPE_KEYS = ("q_rope_sig", "q_rope_noise", "k_rope")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdla.load_library()


def _run(x, window, causal, status=None, scale=0.0):
    return gdla.gdla_attn_fwd_rope(x["q_sig"], x["q_noise"], x["q_rope_sig"], x["q_rope_noise"],
                                   x["k"], x["v"], x["k_rope"], x["lam"], x["gate"],
                                   window=window, causal=causal, d_status=status, scale=scale)


def _check_full(x, out, window, causal, what):
    cpu = {k: v.cpu() for k, v in x.items()}
    ref = oracle.gdla_attn(cpu["q_sig"], cpu["q_noise"], cpu["k"], cpu["v"], cpu["lam"],
                           cpu["gate"], window=window, causal=causal,
                           q_rope_sig=cpu["q_rope_sig"], q_rope_noise=cpu["q_rope_noise"],
                           k_rope=cpu["k_rope"])
    got = out.reshape(ref.shape).float().cpu().numpy()
    return assert_parity(got, ref, what)


def _check_rows(x, out, rows, window, causal, what):
    ref = oracle.gdla_attn_rows(gather_rows(x["q_sig"], rows), gather_rows(x["q_noise"], rows),
                                x["k"].cpu(), x["v"].cpu(), gather_rows(x["lam"], rows),
                                gather_rows(x["gate"], rows), rows, window=window, causal=causal,
                                q_rope_sig_rows=gather_rows(x["q_rope_sig"], rows),
                                q_rope_noise_rows=gather_rows(x["q_rope_noise"], rows),
                                k_rope=x["k_rope"].cpu())
    return assert_parity(gather_rows(out, rows).float().numpy(), ref, what)


EDGE = [
    # B, T, Hs, Hn, Hkv, d, window, causal
    (1, 256, 8, 2, 2, 64, 0, True),      # the tiny shape with the rotary term
    (1, 1, 8, 2, 2, 64, 0, True),        # one token
    (1, 2, 8, 2, 2, 128, 0, True),
    (2, 127, 8, 2, 2, 128, 0, True),     # ragged single tile
    (1, 129, 8, 2, 2, 128, 0, True),     # one row into a second tile
    (1, 300, 4, 4, 4, 128, 0, True),     # g = 1
    (1, 300, 6, 2, 2, 64, 0, True),      # g = 3
    (3, 257, 8, 2, 2, 64, 0, True),
    (1, 700, 8, 2, 2, 128, 1, True),     # window of one key
    (1, 700, 8, 2, 2, 128, 128, True),   # the Motif 3 window
    (1, 700, 8, 2, 2, 64, 200, True),    # window wider than a tile
    (2, 333, 8, 2, 2, 128, 127, True),
    (1, 333, 8, 2, 2, 128, 0, False),    # no mask
    (2, 200, 8, 2, 2, 64, 0, False),
    (1, 1100, 8, 2, 2, 128, 0, True),    # many tiles per head
]


@pytest.mark.parametrize("B,T,Hs,Hn,Hkv,d,window,causal", EDGE)
def test_rope_every_element(B, T, Hs, Hn, Hkv, d, window, causal):
    wl = custom(B, T, Hs, Hn, Hkv, d, window=window, causal=causal, d_rope=64)
    x = make_inputs(wl, seed=T + 7 * window + d, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(x, window, causal, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_full(x, out, window, causal, f"rope edge {B},{T},{Hs},{Hn},{d},{window},{causal}")


@pytest.mark.parametrize("name", ["full_rope", "window_rope"])
def test_rope_workload_sampled_rows(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(x, wl.window, wl.causal, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = sample_rows(wl.B, wl.T, 200, seed=11, extra=range(wl.T - 130, wl.T))
    _check_rows(x, out, rows, wl.window, wl.causal, name)


def test_rope_noise_equal_signal_gives_zero():
    """Q_noise and its rotary query copied into every signal head of the
    group, lambda = 1, G = 1: D = 0, so |O| <= 1e-3."""
    wl = custom(2, 600, 16, 4, 4, 128, window=0, d_rope=64)
    x = make_inputs(wl, seed=5, device="cuda")
    x["q_sig"] = x["q_noise"].repeat_interleave(wl.g, dim=2).contiguous()
    x["q_rope_sig"] = x["q_rope_noise"].repeat_interleave(wl.g, dim=2).contiguous()
    x["lam"] = torch.ones_like(x["lam"])
    x["gate"] = torch.ones_like(x["gate"])
    out = _run(x, 0, True)
    torch.cuda.synchronize()
    gdla.check_status()
    assert out.float().abs().max().item() <= 1e-3


def test_rope_zero_rotary_inputs_match_plain_kernel():
    """Zero rotary queries and keys add nothing to the score: with the same
    scale the result matches gdla_attn_fwd (a different kernel) within the
    tolerance."""
    wl = custom(2, 500, 8, 2, 2, 128, window=0, d_rope=64)
    x = make_inputs(wl, seed=3, device="cuda")
    for k in ROPE_KEYS:
        x[k] = torch.zeros_like(x[k])
    sc = 1.0 / np.sqrt(wl.d)
    a = _run(x, 0, True, scale=sc)
    b = gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                           scale=sc)
    torch.cuda.synchronize()
    gdla.check_status()
    assert_parity(a.float().cpu().numpy(), b.float().cpu().numpy().astype(np.float64),
                  "rope kernel with zero rotary inputs vs gdla_attn_fwd")


def test_rope_deterministic():
    wl = custom(1, 1000, 8, 2, 2, 128, window=0, d_rope=64)
    x = make_inputs(wl, seed=9, device="cuda")
    a = _run(x, 0, True)
    b = _run(x, 0, True)
    torch.cuda.synchronize()
    gdla.check_status()
    assert torch.equal(a, b)
