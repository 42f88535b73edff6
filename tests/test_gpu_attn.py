"""GPU parity of the fused GDLA attention kernel against the float64 oracle.

Every call goes through the C ABI (libgdla.so via the ctypes binding).  Small
shapes are compared on every output element; the workload shapes run at full
size, in the same launch configuration the benchmark times, and are compared
on sampled rows.  Row subsets are exact: an output row depends only on its own
query row and the keys its mask keeps, so the oracle evaluates those rows alone.
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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdla.load_library()


def _run(x, window, causal, status=None, out=None):
    return gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                              window=window, causal=causal, d_status=status, out=out)


def _check_rows(x, out, wl, rows, window, causal, what):
    gdla.check_status()  # calls that passed no status word share the default one
    ref = oracle.gdla_attn_rows(gather_rows(x["q_sig"], rows), gather_rows(x["q_noise"], rows),
                                x["k"].cpu(), x["v"].cpu(), gather_rows(x["lam"], rows),
                                gather_rows(x["gate"], rows), rows, window=window, causal=causal)
    got = gather_rows(out, rows).float().numpy()
    return assert_parity(got, ref, what)


def _check_full(x, out, window, causal, what):
    gdla.check_status()
    cpu = {k: v.cpu() for k, v in x.items()}
    ref = oracle.gdla_attn(cpu["q_sig"], cpu["q_noise"], cpu["k"], cpu["v"], cpu["lam"],
                           cpu["gate"], window=window, causal=causal)
    got = out.reshape(ref.shape).float().cpu().numpy()
    return assert_parity(got, ref, what)


def test_tiny_config_every_element():
    wl = WORKLOADS["tiny"]
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=0).items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(x, 0, True, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_full(x, out, 0, True, "tiny")


@pytest.mark.parametrize("name,n_random", [("window", 300), ("full", 40)])
def test_workload_sampled_rows(name, n_random):
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(x, wl.window, wl.causal, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = sample_rows(wl.B, wl.T, n_random, seed=1)
    _check_rows(x, out, wl, rows, wl.window, wl.causal, name)


@pytest.mark.parametrize("name,n_random", [("long_full", 6), ("long_window", 300)])
def test_long_context_sampled_rows(name, n_random):
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(x, wl.window, wl.causal, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = sample_rows(wl.B, wl.T, n_random, seed=2)
    _check_rows(x, out, wl, rows, wl.window, wl.causal, name)
    del x, out
    torch.cuda.empty_cache()


EDGE = [
    # B, T, Hs, Hn, d, window, causal
    (1, 1, 8, 2, 64, 0, True),
    (1, 2, 8, 2, 128, 0, True),
    (2, 127, 8, 2, 128, 0, True),
    (1, 129, 8, 2, 128, 0, True),
    (1, 300, 4, 4, 128, 0, True),     # g = 1: (noise, signal) only
    (1, 300, 4, 2, 128, 0, True),     # g = 2: three heads, last phase single slot
    (1, 300, 6, 2, 64, 0, True),      # g = 3
    (3, 257, 8, 2, 64, 0, True),
    (1, 700, 8, 2, 128, 1, True),     # W = 1: diagonal only
    (1, 700, 8, 2, 128, 128, True),
    (1, 700, 8, 2, 64, 200, True),
    (1, 700, 8, 2, 128, 700, True),   # W = T
    (1, 700, 8, 2, 128, 705, True),   # W > T
    (1, 333, 8, 2, 128, 0, False),    # no mask
    (2, 200, 8, 2, 64, 0, False),
    (1, 4097, 8, 2, 128, 0, True),
    (1, 4097, 8, 2, 128, 128, True),
    # windows of at most one K/V tile (union-row kernel) and just above it
    (1, 700, 8, 2, 128, 64, True),
    (2, 333, 8, 2, 128, 127, True),
    (1, 700, 8, 2, 128, 129, True),
    (1, 300, 4, 4, 128, 128, True),   # g = 1
    (1, 300, 4, 2, 128, 128, True),   # g = 2
    (1, 300, 6, 2, 64, 128, True),    # g = 3, d = 64
    (3, 257, 8, 2, 64, 100, True),
    (1, 100, 8, 2, 128, 128, True),   # a single query block: no edge tile
]


@pytest.mark.parametrize("B,T,Hs,Hn,d,window,causal", EDGE)
def test_edge_shapes_every_element(B, T, Hs, Hn, d, window, causal):
    wl = custom(B, T, Hs, Hn, Hn, d, window=window, causal=causal)
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=T + d).items()}
    out = _run(x, window, causal)
    torch.cuda.synchronize()
    what = f"edge {B},{T},{Hs},{Hn},{d},{window},{causal}"
    if B * T <= 1500:
        _check_full(x, out, window, causal, what)
    else:  # long ragged shapes: every block edge plus random rows
        rows = sample_rows(B, T, 300, seed=T, extra=range(T - 300, T))
        _check_rows(x, out, wl, rows, window, causal, what)


def test_noise_equal_signal_gives_zero():
    """Q_noise copied into every signal head of its group, lambda=1, G=1: O ~ 0."""
    wl = custom(2, 600, 16, 4, 4, 128, window=0)
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=5).items()}
    x["q_sig"] = x["q_noise"].repeat_interleave(wl.g, dim=2).contiguous()
    x["lam"] = torch.ones_like(x["lam"])
    x["gate"] = torch.ones_like(x["gate"])
    out = _run(x, 0, True)
    torch.cuda.synchronize()
    assert out.float().abs().max().item() <= 1e-3


def test_deterministic_and_stream_ordered():
    wl = custom(2, 1000, 8, 2, 2, 128, window=0)
    x = make_inputs(wl, seed=9, device="cuda")
    a = _run(x, 0, True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b = _run(x, 0, True)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_guard_regions_untouched():
    """Output written exactly in place: canaries on both sides survive."""
    wl = custom(1, 383, 8, 2, 2, 128, window=0)
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=13).items()}
    n = wl.B * wl.T * wl.Hs * wl.d
    guard = 4096
    buf = torch.full((guard + n + guard,), 12345, dtype=torch.int16, device="cuda")
    out = buf[guard:guard + n].view(torch.bfloat16).view(wl.B, wl.T, wl.Hs * wl.d)
    _run(x, 0, True, out=out)
    torch.cuda.synchronize()
    assert bool((buf[:guard] == 12345).all()) and bool((buf[guard + n:] == 12345).all())
    _check_full(x, out, 0, True, "guarded")


def test_rejected_call_enqueues_nothing():
    wl = custom(1, 64, 8, 2, 2, 64)
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=1).items()}
    out = torch.full((1, 64, 8 * 64), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdla.GDLAError):
        gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                           window=-3, out=out)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
