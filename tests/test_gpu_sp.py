"""GPU parity of the sliding window on shards of a sequence (gdla_attn_fwd_sp).

One GPU runs the shards one after another: shard s of a sequence gets the
K/V rows [start - 128, start + T_loc) (its halo, then its own rows), exactly
what the halo exchange gives a rank.  When every shard starts on a multiple
of 128 tokens its output rows equal the unsharded call's bit for bit (same
K/V tiles, same arithmetic); otherwise they are checked against the float64
oracle.  Calls go through the C ABI.
"""
import numpy as np
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
import oracle
from grouped_differential_attention_gdla_b200 import halo
from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, custom, make_inputs
from parity import assert_parity, gather_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdla.load_library()


def _shards(x, T, n_shards, window):
    """Run every shard through gdla_attn_fwd_sp; returns the stitched output."""
    B = x["q_sig"].shape[0]
    bounds = np.linspace(0, T, n_shards + 1).astype(int)
    outs = []
    for s in range(n_shards):
        a, b = int(bounds[s]), int(bounds[s + 1])
        pre = 0 if s == 0 else halo.HALO_ROWS
        sl = lambda t: t[:, a:b].contiguous()
        k = x["k"][:, a - pre:b].contiguous()
        v = x["v"][:, a - pre:b].contiguous()
        outs.append(gdla.gdla_attn_fwd_sp(sl(x["q_sig"]), sl(x["q_noise"]), k, v, sl(x["lam"]),
                                          sl(x["gate"]), window, pre))
    gdla.check_status()
    return torch.cat(outs, dim=1)


@pytest.mark.parametrize("B,T,n_shards,window", [
    (1, 4096, 4, 128), (2, 2048, 2, 128), (1, 3072, 3, 64), (1, 2048, 8, 1)])
def test_aligned_shards_equal_unsharded_bitwise(B, T, n_shards, window):
    wl = custom(B, T, 16, 4, 4, 128, window=window)
    x = make_inputs(wl, seed=T + window, device="cuda")
    ref = gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                             window=window)
    got = _shards(x, T, n_shards, window)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("B,T,n_shards,window", [(1, 2000, 3, 128), (2, 1100, 2, 100)])
def test_ragged_shards_match_the_oracle(B, T, n_shards, window):
    wl = custom(B, T, 8, 2, 2, 128, window=window)
    x = make_inputs(wl, seed=T, device="cuda")
    got = _shards(x, T, n_shards, window)
    torch.cuda.synchronize()
    cpu = {k: v.cpu() for k, v in x.items()}
    ref = oracle.gdla_attn(cpu["q_sig"], cpu["q_noise"], cpu["k"], cpu["v"], cpu["lam"],
                           cpu["gate"], window=window)
    assert_parity(got.reshape(ref.shape).float().cpu().numpy(), ref, f"sp shards {B},{T}")


def test_long_window_layer_in_eight_shards_sampled_rows():
    """The W=128, T=262144 layer split into 8 shards of 32768 tokens."""
    wl = WORKLOADS["long_window"]
    x = make_inputs(wl, seed=0, device="cuda")
    got = _shards(x, wl.T, 8, wl.window)
    torch.cuda.synchronize()
    T_loc = wl.T // 8
    rows = np.unique(np.concatenate([np.arange(s * T_loc - 2, s * T_loc + 130)
                                     for s in range(1, 8)] + [np.arange(0, 130)]))
    ref = oracle.gdla_attn_rows(gather_rows(x["q_sig"], rows), gather_rows(x["q_noise"], rows),
                                x["k"].cpu(), x["v"].cpu(), gather_rows(x["lam"], rows),
                                gather_rows(x["gate"], rows), rows, window=wl.window)
    assert_parity(gather_rows(got, rows).float().numpy(), ref, "long_window, 8 shards")


def test_sp_rejects_wide_windows_and_bad_prefix():
    wl = custom(1, 256, 8, 2, 2, 64, window=128)
    x = make_inputs(wl, seed=1, device="cuda")
    kv = torch.cat([x["k"][:, :128], x["k"]], dim=1)
    args = (x["q_sig"], x["q_noise"], kv, kv, x["lam"], x["gate"])
    with pytest.raises(gdla.GDLAError):
        gdla.gdla_attn_fwd_sp(*args, 129, 128)
    with pytest.raises(gdla.GDLAError):
        gdla.gdla_attn_fwd_sp(x["q_sig"], x["q_noise"], x["k"], x["k"], x["lam"], x["gate"],
                              0, 0)
