"""GPU parity of the fused RMSNorm + W^KV_b expand kernel, and of the whole
latent-KV path (expand then attention) against the float64 oracle chained the
same way.  Calls go through the C ABI.  The oracle chain keeps K and V in
float64; the GPU rounds them to bf16 between the two kernels, which the
per-tensor tolerance absorbs (max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3).
"""
import numpy as np
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
import oracle
from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, make_inputs
from parity import assert_parity, gather_rows, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdla.load_library()


def _oracle_kv(c_kv_rows, w, rms_w, eps, hkv, dh):
    chat = oracle.rmsnorm(c_kv_rows, rms_w, eps)
    return oracle.kv_expand(chat, w, hkv, dh, dh)


@pytest.mark.parametrize("n,dl,hkv,dh,with_w", [
    (1, 512, 16, 128, False),
    (300, 512, 16, 128, True),
    (129, 64, 3, 128, False),
    (257, 256, 2, 64, True),
    (1000, 512, 1, 64, False),
    (4096, 448, 5, 128, True),
])
def test_expand_every_element(n, dl, hkv, dh, with_w):
    g = torch.Generator().manual_seed(n + dl)
    c = torch.randn(n, dl, generator=g).to(torch.bfloat16)
    w = (torch.randn(dl, hkv * 2 * dh, generator=g) / dl ** 0.5).to(torch.bfloat16)
    rw = (torch.rand(dl, generator=g) + 0.5).to(torch.bfloat16) if with_w else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    k, v = gdla.gdla_kv_expand(c.cuda(), w.cuda(), rw.cuda() if rw is not None else None,
                               eps=1e-6, d_head=dh, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rk, rv = _oracle_kv(c, w, rw, 1e-6, hkv, dh)
    shape = f"n={n} dl={dl} Hkv={hkv} d={dh}"
    assert_parity(k.float().cpu().numpy(), rk, f"expand K {shape}")
    assert_parity(v.float().cpu().numpy(), rv, f"expand V {shape}")


def test_latent_config_expand_sampled_tokens():
    wl = WORKLOADS["latent"]
    x = make_inputs(wl, seed=0, device="cuda")
    k, v = gdla.gdla_kv_expand(x["c_kv"], x["w_kvb"], None, eps=wl.eps, d_head=wl.d)
    torch.cuda.synchronize()
    n = wl.B * wl.T
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(0, 130), np.arange(n - 130, n),
                                     rng.integers(0, n, 500)]))
    idx = torch.as_tensor(rows, device="cuda")
    rk, rv = _oracle_kv(x["c_kv"].index_select(0, idx).cpu(), x["w_kvb"].cpu(), None, wl.eps,
                        wl.Hkv, wl.d)
    assert_parity(k.index_select(0, idx).float().cpu().numpy(), rk, "K (latent config)")
    assert_parity(v.index_select(0, idx).float().cpu().numpy(), rv, "V (latent config)")


def test_latent_config_chained_attention():
    """c_KV -> RMSNorm -> W^KV_b -> GDLA attention, all on the GPU, against the
    oracle chain in float64 on sampled rows."""
    wl = WORKLOADS["latent"]
    x = make_inputs(wl, seed=0, device="cuda")
    k, v = gdla.gdla_kv_expand(x["c_kv"], x["w_kvb"], None, eps=wl.eps, d_head=wl.d)
    out = gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"], k.view(wl.B, wl.T, wl.Hkv, wl.d),
                             v.view(wl.B, wl.T, wl.Hkv, wl.d), x["lam"], x["gate"],
                             window=wl.window, causal=wl.causal)
    torch.cuda.synchronize()
    # every query block's first and last rows up to token 8191, block edges
    # across the sequence and random rows: 256+ rows, keys up to the last one
    rows = sample_rows(wl.B, wl.T, 140, seed=4,
                       extra=[q + o for q in range(0, 8192, 128) for o in (0, 127)])
    assert rows.size >= 256
    t_max = int(rows.max()) + 1
    rk, rv = _oracle_kv(x["c_kv"][:t_max].cpu(), x["w_kvb"].cpu(), None, wl.eps, wl.Hkv, wl.d)
    ref = oracle.gdla_attn_rows(gather_rows(x["q_sig"], rows), gather_rows(x["q_noise"], rows),
                                rk.reshape(1, t_max, wl.Hkv, wl.d),
                                rv.reshape(1, t_max, wl.Hkv, wl.d),
                                gather_rows(x["lam"], rows), gather_rows(x["gate"], rows), rows,
                                window=wl.window, causal=wl.causal)
    assert_parity(gather_rows(out, rows).float().numpy(), ref, "latent chain")
