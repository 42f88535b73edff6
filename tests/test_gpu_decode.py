"""GPU parity of the decode over the KV latent cache against the float64 oracle.

The GPU path is the cache write (gdla_latent_rmsnorm of each token's KV
latent) followed by gdla_decode_fwd for the newest token of every sequence;
the oracle takes the raw latents and applies RMSNorm, the W^KV_b expand and
the forward pass for that token as written ("Motif 3: Technical Report",
paper.rainbus.top, step 2 and its "technical novelty" paragraph).  Calls go
through the C ABI.  Tolerance per tensor: 1e-2 * max|oracle| + 1e-3.
"""
import numpy as np
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
import oracle
from parity import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdla.load_library()


def _case(B, L_max, Hs, Hn, d, dl, seed, with_w=False):
    g = torch.Generator(device="cuda").manual_seed(seed)
    bf = lambda *shape, s=1.0: (torch.randn(*shape, generator=g, device="cuda") * s).to(
        torch.bfloat16)
    x = {
        "q_sig": bf(B, Hs, d), "q_noise": bf(B, Hn, d), "c_kv": bf(B, L_max, dl),
        "w_kvb": bf(dl, Hn * 2 * d, s=dl ** -0.5),
        "lam": torch.sigmoid(torch.randn(B, Hs, generator=g, device="cuda")).to(torch.bfloat16),
        "gate": torch.sigmoid(torch.randn(B, Hs * d, generator=g, device="cuda")).to(
            torch.bfloat16),
    }
    x["rms_w"] = (torch.rand(dl, generator=g, device="cuda") + 0.5).to(torch.bfloat16) \
        if with_w else None
    return x


def _decode(x, lens, window, workspace=None, status=None):
    c_hat = gdla.gdla_latent_rmsnorm(x["c_kv"], x["rms_w"], 1e-6)
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return gdla.gdla_decode_fwd(x["q_sig"], x["q_noise"], c_hat, cl, x["w_kvb"], x["lam"],
                                x["gate"], window=window, workspace=workspace, d_status=status)


def _oracle(x, lens, window):
    cpu = lambda t: None if t is None else t.cpu()
    return oracle.decode(cpu(x["q_sig"]), cpu(x["q_noise"]), cpu(x["c_kv"]), lens,
                         cpu(x["w_kvb"]), cpu(x["lam"]), cpu(x["gate"]), rms_w=cpu(x["rms_w"]),
                         window=window)


@pytest.mark.parametrize("B,L_max,Hs,Hn,d,dl,lens,window,with_w", [
    (3, 300, 8, 2, 64, 512, [300, 1, 129], 0, False),
    (3, 300, 8, 2, 64, 512, [300, 1, 129], 128, True),
    (2, 700, 8, 2, 128, 256, [700, 385], 5, False),
    (4, 2000, 64, 16, 128, 512, [2000, 1, 777, 1024], 0, False),
    (4, 2000, 64, 16, 128, 512, [2000, 1, 777, 1024], 128, True),
    (2, 5000, 64, 16, 128, 512, [5000, 3000], 1, False),
    # one signal head per group (2 head rows per group in the merge and output)
    (5, 600, 4, 4, 128, 512, [600, 1, 250, 599, 128], 0, False),
    # three signal heads per group, d = 64, a 256-d latent
    (3, 400, 6, 2, 64, 256, [400, 17, 256], 0, True),
    # eight signal heads per group (9 head rows per group, 80 padded rows)
    (2, 300, 16, 2, 128, 512, [300, 77], 64, False),
    # 37 sequences: several sequences per output-GEMM CTA, the last block ragged
    (37, 300, 64, 16, 128, 512, [300 - 8 * i for i in range(37)], 0, False),
])
def test_decode_matches_oracle(B, L_max, Hs, Hn, d, dl, lens, window, with_w):
    x = _case(B, L_max, Hs, Hn, d, dl, seed=L_max + window, with_w=with_w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _decode(x, lens, window, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_parity(out.float().cpu().numpy(), _oracle(x, lens, window),
                  f"decode B={B} L={L_max} {Hs}/{Hn} d={d} dl={dl} W={window}")


def test_decode_long_cache_window_and_full_sampled():
    """64 sequences over a 32768-token cache: every sequence with a window of
    128, and 4 of them over all their keys."""
    B, L_max = 64, 32768
    x = _case(B, L_max, 64, 16, 128, 512, seed=7)
    rng = np.random.default_rng(1)
    lens = [L_max, 1, 128, 129] + rng.integers(1, L_max + 1, B - 4).tolist()
    out = _decode(x, lens, 128)
    torch.cuda.synchronize()
    gdla.check_status()
    assert_parity(out.float().cpu().numpy(), _oracle(x, lens, 128), "decode 64 x 32768, W=128")
    sub = {k: (v[:4] if k not in ("w_kvb", "rms_w") and v is not None else v)
           for k, v in x.items()}
    sub["c_kv"] = sub["c_kv"][:, :4096].contiguous()
    lens4 = [4096, 1, 2049, 3333]
    out4 = _decode(sub, lens4, 0)
    torch.cuda.synchronize()
    assert_parity(out4.float().cpu().numpy(), _oracle(sub, lens4, 0), "decode 4 x 4096, full")


def test_latent_rmsnorm_every_element():
    x = _case(2, 333, 8, 2, 64, 512, seed=3, with_w=True)
    got = gdla.gdla_latent_rmsnorm(x["c_kv"], x["rms_w"], 1e-6)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(x["c_kv"].reshape(-1, 512).cpu(), x["rms_w"].cpu(), 1e-6)
    assert_parity(got.reshape(-1, 512).float().cpu().numpy(), ref, "latent rmsnorm")


def test_decode_reused_workspace_and_rows_past_the_length():
    """Two calls sharing one workspace give the same bits; finite values in
    cache rows past each length change nothing."""
    B, L_max = 3, 1000
    x = _case(B, L_max, 64, 16, 128, 512, seed=11)
    lens = [1000, 400, 1]
    ws = torch.empty(gdla.gdla_decode_workspace_bytes(B, L_max, 64, 16, 512, 0),
                     dtype=torch.uint8, device="cuda")
    a = _decode(x, lens, 0, workspace=ws).clone()
    b = _decode(x, lens, 0, workspace=ws).clone()
    x2 = dict(x)
    x2["c_kv"] = x["c_kv"].clone()
    x2["c_kv"][1, 400:] = 30.0
    x2["c_kv"][2, 1:] = -7.0
    c = _decode(x2, lens, 0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(a, c)


def test_decode_cache_len_out_of_range_sets_status():
    x = _case(2, 256, 8, 2, 64, 512, seed=2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _decode(x, [0, 300], 0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == gdla._binding.GDLA_ERR_INVALID_ARG


def test_decode_graph_replay_matches_eager():
    """A decode step captured once in a CUDA graph (as a serving loop, and the
    benchmark, replay it) gives, for new queries copied into the captured
    buffers, bit for bit the output of an eager call on those queries."""
    B, L_max = 6, 1000
    lens = [1000, 1, 517, 128, 129, 900]
    x = _case(B, L_max, 64, 16, 128, 512, seed=21)
    c_hat = gdla.gdla_latent_rmsnorm(x["c_kv"], None, 1e-6)
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(gdla.gdla_decode_workspace_bytes(B, L_max, 64, 16, 512, 0),
                     dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_sig, q_noise = x["q_sig"].clone(), x["q_noise"].clone()
    out = torch.empty(B, 64 * 128, dtype=torch.bfloat16, device="cuda")

    def call(o, qs, qn):
        gdla.gdla_decode_fwd(qs, qn, c_hat, cl, x["w_kvb"], x["lam"], x["gate"], out=o,
                             workspace=ws, d_status=status,
                             stream=torch.cuda.current_stream())

    call(out, q_sig, q_noise)  # one-time kernel set-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(out, q_sig, q_noise)
    g = torch.Generator(device="cuda").manual_seed(5)
    for _ in range(2):
        new_s = torch.randn(q_sig.shape, generator=g, device="cuda").to(torch.bfloat16)
        new_n = torch.randn(q_noise.shape, generator=g, device="cuda").to(torch.bfloat16)
        q_sig.copy_(new_s)
        q_noise.copy_(new_n)
        graph.replay()
        torch.cuda.synchronize()
        replayed = out.clone()
        eager = torch.empty_like(out)
        call(eager, new_s, new_n)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(replayed, eager)
    del graph
