"""gdla_decode_fwd_noalloc: the decode for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc (a host framework that
owns the allocator and forbids allocation inside its callbacks, a plugin with
no allocator handle, a serving loop that must not allocate between requests),
so they cannot supply the workspace gdla_decode_fwd needs.  The no-alloc entry
point takes the same inputs and outputs and uses a scratch array compiled into
libgdla.so instead.  These tests call it through the C ABI and hold it to the
existing entry point's results, within the tolerance every parity test here
uses (1e-2 * max|reference| + 1e-3), on two calls in a row; the second call
runs on other inputs, so stale scratch contents from the first would show.

The file is named to be collected last: the GPU test must also pass after
every other test has run in the same process.
"""
import ctypes

import numpy as np
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
from grouped_differential_attention_gdla_b200 import _binding

RTOL, ATOL = 1e-2, 1e-3


def _lib_or_skip():
    try:
        from grouped_differential_attention_gdla_b200.build import build
        build()
        return gdla.load_library()
    except Exception as exc:  # nvcc missing on this host
        pytest.skip(f"libgdla.so unavailable: {exc}")


def test_oversized_request_refused_before_touching_the_device():
    """A shape whose workspace exceeds the compiled-in array is refused with
    GDLA_ERR_UNSUPPORTED, before any device call (this runs without a GPU)."""
    lib = _lib_or_skip()
    B, L_max, Hs, Hn, d, dl = 64, 32768, 64, 16, 128, 512
    need = gdla.gdla_decode_workspace_bytes(B, L_max, Hs, Hn, dl, 0)
    assert need > _binding.DECODE_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    rc = lib.gdla_decode_fwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, B, L_max,
                                     Hs, Hn, Hn, d, dl, 0, 0.0, None, None)
    assert rc == _binding.GDLA_ERR_UNSUPPORTED


def _case(B, L_max, Hs, Hn, d, dl, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    bf = lambda *shape, s=1.0: (torch.randn(*shape, generator=g, device="cuda") * s).to(
        torch.bfloat16)
    x = {
        "q_sig": bf(B, Hs, d), "q_noise": bf(B, Hn, d),
        "c_hat": gdla.gdla_latent_rmsnorm(bf(B, L_max, dl), None, 1e-6),
        "w_kvb": bf(dl, Hn * 2 * d, s=dl ** -0.5),
        "lam": torch.sigmoid(torch.randn(B, Hs, generator=g, device="cuda")).to(torch.bfloat16),
        "gate": torch.sigmoid(torch.randn(B, Hs * d, generator=g, device="cuda")).to(
            torch.bfloat16),
    }
    return x


def _close(got, ref, what):
    got = got.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    err = float(np.abs(got - ref).max())
    tol = RTOL * float(np.abs(ref).max()) + ATOL
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err <= tol, f"{what}: max|noalloc - workspace| = {err:.3e} > tol {tol:.3e}"


@pytest.mark.gpu
@pytest.mark.parametrize("B,L_max,Hs,Hn,d,dl,lens,window", [
    (4, 2000, 64, 16, 128, 512, [2000, 1, 777, 1024], 0),
    (3, 4096, 64, 16, 128, 512, [4096, 130, 3000], 128),
])
def test_noalloc_matches_workspace_entry_point_twice(B, L_max, Hs, Hn, d, dl, lens, window):
    _lib_or_skip()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, seed in enumerate((11, 12)):
        x = _case(B, L_max, Hs, Hn, d, dl, seed + window)
        args = (x["q_sig"], x["q_noise"], x["c_hat"], cl, x["w_kvb"], x["lam"], x["gate"])
        ref = gdla.gdla_decode_fwd(*args, window=window)
        out = torch.empty((B, Hs * d), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        gdla.gdla_decode_fwd_noalloc(*args, out, window=window, d_status=status)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before, "the no-alloc call allocated"
        assert int(status.item()) == 0
        _close(out, ref, f"call {call + 1}, B={B} L={L_max} W={window}")
