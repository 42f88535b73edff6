"""The C-ABI library on the host: it loads, exports every entry point that
include/gdla.h declares, and rejects bad arguments with the documented status
before touching CUDA (no GPU is needed for any call made here)."""
import ctypes
import os
import re

import pytest

import grouped_differential_attention_gdla_b200 as gdla
from grouped_differential_attention_gdla_b200 import _binding
from grouped_differential_attention_gdla_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdla.h")

OK, INVALID, UNSUPPORTED, ALIGN = 0, -1, -2, -3
A = 0x100000  # a 16-byte aligned fake device address; never dereferenced here
M = 0x100008  # misaligned fake address


@pytest.fixture(scope="module")
def lib():
    build()
    return gdla.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdla_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert set(declared) == {"gdla_version", "gdla_status_string", "gdla_kv_expand",
                             "gdla_attn_fwd", "gdla_attn_fwd_sp", "gdla_latent_rmsnorm",
                             "gdla_decode_workspace_bytes", "gdla_decode_fwd",
                             "gdla_selftest_wait_timeout", "gdla_decode_fwd_noalloc",
                             "gdla_attn_fwd_rope", "gdla_attn_bwd_workspace_bytes",
                             "gdla_attn_bwd"}
    for name in declared:
        assert hasattr(lib, name), f"{name} missing from libgdla.so"
    assert set(declared) == set(_binding.EXPORTED)


def test_version_and_status_strings(lib):
    assert gdla.gdla_version() >= 100
    for code in (0, -1, -2, -3, -4, -5):
        s = gdla.gdla_status_string(code)
        assert s and s != "unknown status code"
    assert gdla.gdla_status_string(7) == "unknown status code"


def _attn(lib, q=A, qn=A, k=A, v=A, lam=A, gate=A, out=A, B=1, T=256, Hs=8, Hn=2, Hkv=2, d=64,
          window=0, causal=1, scale=0.0, status=None):
    return lib.gdla_attn_fwd(q, qn, k, v, lam, gate, out, B, T, Hs, Hn, Hkv, d, window, causal,
                             ctypes.c_float(scale), status, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(qn=None), INVALID), (dict(k=None), INVALID),
    (dict(v=None), INVALID), (dict(lam=None), INVALID), (dict(gate=None), INVALID),
    (dict(out=None), INVALID), (dict(B=-1), INVALID), (dict(T=-5), INVALID),
    (dict(Hs=0), INVALID), (dict(Hn=0), INVALID), (dict(d=0), INVALID),
    (dict(window=-1), INVALID), (dict(causal=2), INVALID),
    (dict(causal=0, window=4), INVALID), (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID),
    (dict(Hs=6, Hn=4, Hkv=4), UNSUPPORTED), (dict(Hn=2, Hkv=4), UNSUPPORTED),
    (dict(d=32), UNSUPPORTED), (dict(d=96), UNSUPPORTED), (dict(T=2 ** 31), UNSUPPORTED),
    (dict(q=M), ALIGN), (dict(qn=M), ALIGN), (dict(k=M), ALIGN), (dict(v=M), ALIGN),
    (dict(lam=M), ALIGN), (dict(gate=M), ALIGN), (dict(out=M), ALIGN),
    (dict(status=0x100002), ALIGN), (dict(status=0x100001), ALIGN),
    (dict(T=0), OK), (dict(B=0), OK), (dict(T=0, q=None, out=None), OK),
])
def test_attn_argument_errors(lib, kw, code):
    assert _attn(lib, **kw) == code


def _rope(lib, q=A, qn=A, qr=A, qrn=A, k=A, v=A, kr=A, lam=A, gate=A, out=A, B=1, T=256, Hs=8,
          Hn=2, Hkv=2, d=64, dr=64, window=0, causal=1, scale=0.0, status=None):
    return lib.gdla_attn_fwd_rope(q, qn, qr, qrn, k, v, kr, lam, gate, out, B, T, Hs, Hn, Hkv, d,
                                  dr, window, causal, ctypes.c_float(scale), status, None)


@pytest.mark.parametrize("kw,code", [
    (dict(qr=None), INVALID), (dict(qrn=None), INVALID), (dict(kr=None), INVALID),
    (dict(q=None), INVALID), (dict(dr=-64), INVALID), (dict(causal=0, window=3), INVALID),
    (dict(dr=32), UNSUPPORTED), (dict(dr=128), UNSUPPORTED), (dict(d=96), UNSUPPORTED),
    (dict(Hn=2, Hkv=4), UNSUPPORTED),
    (dict(qr=M), ALIGN), (dict(qrn=M), ALIGN), (dict(kr=M), ALIGN), (dict(q=M), ALIGN),
    (dict(status=0x100002), ALIGN),
    (dict(T=0), OK), (dict(B=0), OK),
    # d_rope = 0 ignores the rotary pointers and validates like gdla_attn_fwd
    (dict(dr=0, qr=None, qrn=None, kr=None, out=None), INVALID),
    (dict(dr=0, qr=None, qrn=None, kr=None, B=0), OK),
])
def test_rope_argument_errors(lib, kw, code):
    assert _rope(lib, **kw) == code


def _bwd(lib, q=A, qn=A, k=A, v=A, lam=A, gate=A, do=A, dqs=A, dqn=A, dk=A, dv=A, dl=A, dg=A,
         B=1, T=256, Hs=8, Hn=2, Hkv=2, d=64, window=0, causal=1, scale=0.0, ws=A,
         ws_bytes=1 << 40, status=None):
    return lib.gdla_attn_bwd(q, qn, k, v, lam, gate, do, dqs, dqn, dk, dv, dl, dg, B, T, Hs, Hn,
                             Hkv, d, window, causal, ctypes.c_float(scale), ws, ws_bytes, status,
                             None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(do=None), INVALID), (dict(dk=None), INVALID),
    (dict(dg=None), INVALID), (dict(ws=None), INVALID), (dict(B=-1), INVALID),
    (dict(window=-1), INVALID), (dict(causal=0, window=3), INVALID),
    (dict(scale=float("nan")), INVALID), (dict(ws_bytes=1024), INVALID),
    (dict(Hs=6, Hn=4, Hkv=4), UNSUPPORTED), (dict(Hs=18, Hn=2, Hkv=2), UNSUPPORTED),
    (dict(d=96), UNSUPPORTED), (dict(Hn=2, Hkv=4), UNSUPPORTED),
    (dict(q=M), ALIGN), (dict(do=M), ALIGN), (dict(dv=M), ALIGN), (dict(ws=M), ALIGN),
    (dict(status=0x100002), ALIGN),
    (dict(T=0), OK), (dict(B=0), OK),
])
def test_bwd_argument_errors(lib, kw, code):
    assert _bwd(lib, **kw) == code


def test_bwd_workspace_size_follows_the_shapes(lib):
    f = lib.gdla_attn_bwd_workspace_bytes
    up = lambda x: (x + 255) // 256 * 256
    # B=2, T=300 (padded to 384 for the statistics), 8 + 2 heads, d=64
    rows, h80, tp = 600, 10, 384
    want = up(up(up(rows * h80 * 64 * 4) + 2 * h80 * tp * 4) + 2 * h80 * tp * 4) + \
        rows * h80 * 64 * 2
    assert f(2, 300, 8, 2, 64) == up(want)
    assert f(0, 300, 8, 2, 64) == 0 and f(2, 0, 8, 2, 64) == 0


def _expand(lib, c=A, w=None, wk=A, eps=1e-6, k=A, v=A, n=300, dl=512, hkv=16, dh=128,
            status=None):
    return lib.gdla_kv_expand(c, w, wk, ctypes.c_float(eps), k, v, n, dl, hkv, dh, status, None)


@pytest.mark.parametrize("kw,code", [
    (dict(c=None), INVALID), (dict(wk=None), INVALID), (dict(k=None), INVALID),
    (dict(v=None), INVALID), (dict(n=-1), INVALID), (dict(dl=0), INVALID),
    (dict(hkv=0), INVALID), (dict(dh=0), INVALID), (dict(eps=-1e-6), INVALID),
    (dict(eps=float("nan")), INVALID), (dict(eps=float("inf")), INVALID),
    (dict(dl=100), UNSUPPORTED), (dict(dl=576), UNSUPPORTED), (dict(dh=96), UNSUPPORTED),
    (dict(n=2 ** 31), UNSUPPORTED),
    (dict(c=M), ALIGN), (dict(wk=M), ALIGN), (dict(k=M), ALIGN), (dict(v=M), ALIGN),
    (dict(w=M), ALIGN), (dict(status=0x100002), ALIGN),
    (dict(n=0), OK), (dict(n=0, c=None), OK),
])
def test_expand_argument_errors(lib, kw, code):
    assert _expand(lib, **kw) == code


def test_binding_rejects_host_tensors():
    import torch
    x = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdla.gdla_attn_fwd(x, x[:, :, :1], x[:, :, :1], x[:, :, :1],
                           torch.zeros(1, 4, 2, dtype=torch.bfloat16),
                           torch.zeros(1, 4, 128, dtype=torch.bfloat16))


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="libgdla.so not found"):
        gdla.load_library(str(tmp_path / "libgdla.so"))


@pytest.mark.parametrize("status,limit,code", [
    (None, 1000, INVALID), (A, 0, INVALID), (A, -5, INVALID), (A, 2 * 10 ** 9, INVALID),
    (0x100002, 1000, ALIGN),
])
def test_selftest_argument_errors(lib, status, limit, code):
    assert lib.gdla_selftest_wait_timeout(status, limit, None) == code


def _sp(lib, q=A, qn=A, k=A, v=A, lam=A, gate=A, out=A, B=1, T=256, kv_prefix=128, Hs=8, Hn=2,
        Hkv=2, d=64, window=128, scale=0.0, status=None):
    return lib.gdla_attn_fwd_sp(q, qn, k, v, lam, gate, out, B, T, kv_prefix, Hs, Hn, Hkv, d,
                                window, ctypes.c_float(scale), status, None)


@pytest.mark.parametrize("kw,code", [
    (dict(kv_prefix=64), INVALID), (dict(kv_prefix=-128), INVALID), (dict(kv_prefix=256), INVALID),
    (dict(window=0), INVALID), (dict(window=129), INVALID), (dict(window=-1), INVALID),
    (dict(window=129, kv_prefix=0), INVALID), (dict(window=0, kv_prefix=0), INVALID),
    (dict(k=None), INVALID), (dict(out=None), INVALID), (dict(T=-1), INVALID),
    (dict(Hn=2, Hkv=4), UNSUPPORTED), (dict(d=96), UNSUPPORTED),
    (dict(T=2 ** 31 - 200), UNSUPPORTED),
    (dict(k=M), ALIGN), (dict(v=M), ALIGN), (dict(status=0x100002), ALIGN),
    (dict(T=0), OK), (dict(B=0), OK),
])
def test_sp_argument_errors(lib, kw, code):
    assert _sp(lib, **kw) == code


WS = 1 << 30  # a workspace size larger than any case below needs


def _dec(lib, q=A, qn=A, c=A, cl=A, w=A, lam=A, gate=A, out=A, B=2, L=300, Hs=8, Hn=2, Hkv=2,
         d=64, dl=512, window=0, scale=0.0, ws=A, ws_bytes=WS, status=None):
    return lib.gdla_decode_fwd(q, qn, c, cl, w, lam, gate, out, B, L, Hs, Hn, Hkv, d, dl, window,
                               ctypes.c_float(scale), ws, ws_bytes, status, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(c=None), INVALID), (dict(cl=None), INVALID),
    (dict(w=None), INVALID), (dict(out=None), INVALID), (dict(ws=None), INVALID),
    (dict(B=-1), INVALID), (dict(L=0), INVALID), (dict(Hs=0), INVALID), (dict(d=0), INVALID),
    (dict(dl=0), INVALID), (dict(window=-1), INVALID), (dict(scale=float("nan")), INVALID),
    (dict(ws_bytes=1000), INVALID),
    (dict(Hn=2, Hkv=4), UNSUPPORTED), (dict(Hs=6, Hn=4, Hkv=4), UNSUPPORTED),
    (dict(Hs=18, Hn=2, Hkv=2), UNSUPPORTED),   # 10 signal heads per group
    (dict(Hs=72, Hn=9, Hkv=9), UNSUPPORTED),   # 81 head rows: more than 80
    (dict(d=96), UNSUPPORTED), (dict(dl=448), UNSUPPORTED), (dict(dl=640), UNSUPPORTED),
    (dict(B=70000), UNSUPPORTED),
    (dict(c=M), ALIGN), (dict(ws=M), ALIGN), (dict(out=M), ALIGN), (dict(cl=0x100002), ALIGN),
    (dict(status=0x100002), ALIGN),
    (dict(B=0), OK), (dict(B=0, q=None), OK),
])
def test_decode_argument_errors(lib, kw, code):
    assert _dec(lib, **kw) == code


def test_decode_workspace_size_follows_the_shapes(lib):
    f = lib.gdla_decode_workspace_bytes
    # 64 sequences x 32768 tokens (256 chunks each), 64 + 16 heads: 9 splits of
    # 29 chunks, 576 CTAs, the fewest waves x (chunks + 3) on 148 SMs
    assert f(64, 32768, 64, 16, 512, 0) == 64 * 80 * 512 * 2 + 64 * 9 * 80 * 514 * 4
    # a 128-token window touches at most 2 chunks: one split per sequence
    assert f(64, 32768, 64, 16, 512, 128) == 64 * 80 * 512 * 2 + 64 * 1 * 80 * 514 * 4
    assert f(1, 100, 8, 2, 512, 0) == 16 * 512 * 2 + 1 * 1 * 16 * 514 * 4
    # 32 + 8 heads: 40 head rows padded to 48
    assert f(1, 100, 32, 8, 512, 0) == 48 * 512 * 2 + 1 * 1 * 48 * 514 * 4
    assert f(0, 100, 8, 2, 512, 0) == 0 and f(1, 0, 8, 2, 512, 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(c=None), INVALID), (dict(out=None), INVALID), (dict(n=-1), INVALID),
    (dict(dl=0), INVALID), (dict(eps=-1.0), INVALID), (dict(eps=float("nan")), INVALID),
    (dict(dl=100), UNSUPPORTED), (dict(c=M), ALIGN), (dict(out=M), ALIGN), (dict(w=M), ALIGN),
    (dict(n=0), OK),
])
def test_latent_rmsnorm_argument_errors(lib, kw, code):
    args = dict(c=A, w=None, eps=1e-6, out=A, n=100, dl=512)
    args.update(kw)
    assert lib.gdla_latent_rmsnorm(args["c"], args["w"], ctypes.c_float(args["eps"]), args["out"],
                                   args["n"], args["dl"], None, None) == code
