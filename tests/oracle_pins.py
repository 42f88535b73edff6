"""Pins that tie the float64 oracle to facts fixed outside the oracle.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with a value derived by hand, a closed form, a library
routine (torch SDPA / rms_norm / matmul in float64) or an invariant that the
GDLA forward must satisfy.  The operation is the one on the page
"Motif 3: Technical Report" (paper.rainbus.top digest), step 2 "GDLA forward";
head counts, window and lambda bounds come from the same page and from
"Вышла новая модель Motif 3" (pikabu.ru).

The pins are plain functions so that tests/test_oracle_mutants.py can run them
against deliberately broken copies of the oracle.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

from grouped_differential_attention_gdla_b200.inputs import custom, make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _f64(t):
    return t.to(torch.float64) if isinstance(t, torch.Tensor) else torch.as_tensor(t, dtype=torch.float64)


def _small(B=2, T=19, Hs=8, Hn=2, Hkv=2, d=16, seed=3, window=0, causal=True):
    wl = custom(B, T, Hs, Hn, Hkv, d, window=window, causal=causal)
    return wl, make_inputs(wl, seed=seed)


def _close(a, b, rtol=1e-11, atol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.abs(a - b).max() if a.size else 0.0
    tol = atol + rtol * (np.abs(b).max() if b.size else 0.0)
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.3e}"


def _sdpa(q, k, v, group, window, causal, scale):
    """torch SDPA in float64 on CPU with KV heads repeated per group."""
    q = _f64(q).permute(0, 2, 1, 3)
    k = _f64(k).repeat_interleave(group, dim=2).permute(0, 2, 1, 3)
    v = _f64(v).repeat_interleave(group, dim=2).permute(0, 2, 1, 3)
    T = q.shape[2]
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    if causal:
        keep = j <= i
        if window > 0:
            keep = keep & (j > i - window)
    else:
        keep = torch.ones(T, T, dtype=torch.bool)
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=scale)
    return out.permute(0, 2, 1, 3)  # [B,T,H,d]


# ---------------------------------------------------------------- golden values

def pin_hand_example(o):
    """Two-token case derived by hand (tests/golden/hand_example.json)."""
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        g = json.load(f)
    ln3 = math.log(3.0)
    k = [[[[ln3 if x == "LN3" else x for x in hd] for hd in tok] for tok in b] for b in g["k"]]
    args = dict(q_sig=np.array(g["q_sig"]), q_noise=np.array(g["q_noise"]), k=np.array(k),
                v=np.array(g["v"]), lam=np.array(g["lam"]), gate=np.array(g["gate"]),
                scale=g["shape"]["scale"])
    _close(o.gdla_attn(**args, window=0, causal=True), g["expected"]["causal"], what="causal")
    _close(o.gdla_attn(**args, window=1, causal=True), g["expected"]["window1"], what="W=1")
    _close(o.gdla_attn(**args, window=0, causal=False), g["expected"]["noncausal"],
           what="non-causal")
    hs = o.attention_path(args["q_sig"], args["k"], args["v"], scale=1.0, rows=[1])
    hn = o.attention_path(args["q_noise"], args["k"], args["v"], scale=1.0, rows=[1])
    _close(hs[0], g["expected_paths_row1_causal"]["H_S"], what="H_S row 1")
    _close(hn[0], g["expected_paths_row1_causal"]["H_N"], what="H_N row 1")


# ---------------------------------------------------------------- closed forms

def pin_first_row_closed_form(o):
    """Row i=0 sees one key: O = G * (1 - lambda) * V[b, 0, h//g]."""
    wl, x = _small()
    out = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    out = out.reshape(wl.B, wl.T, wl.Hs, wl.d)
    v0 = _f64(x["v"])[:, 0].repeat_interleave(wl.g, dim=1)           # [B,Hs,d]
    lam = _f64(x["lam"])[:, 0].unsqueeze(-1)                           # [B,Hs,1]
    gate = _f64(x["gate"])[:, 0].reshape(wl.B, wl.Hs, wl.d)
    _close(out[:, 0], (gate * (1 - lam) * v0).numpy(), what="row 0")


def pin_window_one_closed_form(o):
    """W=1 keeps only the diagonal: O[i] = G * (1 - lambda) * V[i, h//g]."""
    wl, x = _small(window=1)
    out = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], window=1)
    out = out.reshape(wl.B, wl.T, wl.Hs, wl.d)
    v = _f64(x["v"]).repeat_interleave(wl.g, dim=2)
    lam = _f64(x["lam"]).unsqueeze(-1)
    gate = _f64(x["gate"]).reshape(wl.B, wl.T, wl.Hs, wl.d)
    _close(out, (gate * (1 - lam) * v).numpy(), what="W=1")


def pin_equal_keys_mean(o):
    """Equal key rows give uniform weights: H = mean of V over the kept keys."""
    for window, causal in ((0, True), (4, True), (0, False)):
        wl, x = _small(T=13, window=window, causal=causal)
        k = x["k"].clone()
        k[:] = k[:, :1]                                   # every key row = key 0
        T = wl.T
        v = _f64(x["v"])                                  # [B,T,Hkv,d]
        mean = torch.empty_like(v)
        for i in range(T):
            lo = 0 if not causal else (max(0, i - window + 1) if window > 0 else 0)
            hi = T - 1 if not causal else i
            mean[:, i] = v[:, lo:hi + 1].mean(dim=1)
        mean_s = mean.repeat_interleave(wl.g, dim=2)
        lam = _f64(x["lam"]).unsqueeze(-1)
        gate = _f64(x["gate"]).reshape(wl.B, T, wl.Hs, wl.d)
        want = gate * (1 - lam) * mean_s
        got = o.gdla_attn(x["q_sig"], x["q_noise"], k, x["v"], x["lam"], x["gate"],
                          window=window, causal=causal).reshape(wl.B, T, wl.Hs, wl.d)
        _close(got, want.numpy(), rtol=1e-10, what=f"equal keys W={window} causal={causal}")


# ---------------------------------------------------------------- library routines

def pin_lambda0_gate1_is_gqa_sdpa(o):
    """lambda=0, G=1 reduces GDLA to grouped-query attention (torch SDPA)."""
    for window, causal in ((0, True), (5, True), (0, False)):
        wl, x = _small(window=window, causal=causal)
        lam0 = torch.zeros_like(x["lam"])
        gate1 = torch.ones_like(x["gate"])
        got = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], lam0, gate1,
                          window=window, causal=causal)
        want = _sdpa(x["q_sig"], x["k"], x["v"], wl.g, window, causal, 1 / math.sqrt(wl.d))
        _close(got, want.reshape(wl.B * wl.T, -1).numpy(), rtol=1e-10,
               what=f"GQA W={window} causal={causal}")


def pin_differential_matches_sdpa_paths(o):
    """Full combine against two SDPA calls: O = G*(SDPA_S - lambda*Repeat_g(SDPA_N))."""
    for window, causal in ((0, True), (7, True), (0, False)):
        wl, x = _small(T=23, window=window, causal=causal, seed=11)
        sc = 1 / math.sqrt(wl.d)
        hs = _sdpa(x["q_sig"], x["k"], x["v"], wl.g, window, causal, sc)
        hn = _sdpa(x["q_noise"], x["k"], x["v"], 1, window, causal, sc)
        lam = _f64(x["lam"]).unsqueeze(-1)
        gate = _f64(x["gate"]).reshape(wl.B, wl.T, wl.Hs, wl.d)
        want = gate * (hs - lam * hn.repeat_interleave(wl.g, dim=2))
        got = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                          window=window, causal=causal)
        _close(got, want.reshape(wl.B * wl.T, -1).numpy(), rtol=1e-10,
               what=f"GDLA W={window} causal={causal}")
        got_n = o.attention_path(x["q_noise"], x["k"], x["v"], window=window, causal=causal)
        _close(got_n, hn.reshape(wl.B * wl.T, wl.Hn, wl.d).numpy(), rtol=1e-10, what="H_N")


def pin_rmsnorm_matches_torch(o):
    """RMSNorm against torch.nn.functional.rms_norm (float64) and a constant row."""
    g = torch.Generator().manual_seed(5)
    c = torch.randn(37, 512, generator=g, dtype=torch.float32).to(torch.bfloat16)
    w = (torch.rand(512, generator=g) + 0.5).to(torch.bfloat16)
    want = F.rms_norm(_f64(c), (512,), weight=_f64(w), eps=1e-6)
    _close(o.rmsnorm(c, w, 1e-6), want.numpy(), rtol=1e-12, what="rms_norm")
    want1 = F.rms_norm(_f64(c), (512,), weight=None, eps=1e-6)
    _close(o.rmsnorm(c, None, 1e-6), want1.numpy(), rtol=1e-12, what="rms_norm w=1")
    # a constant row a gives a / sqrt(a^2 + eps) in every position
    a = 0.0078125
    const = np.full((2, 512), a)
    const[1] = -a
    got = o.rmsnorm(const, None, 1e-6)
    _close(got[0], np.full(512, a / math.sqrt(a * a + 1e-6)), rtol=1e-13, what="const row")
    _close(got[1], np.full(512, -a / math.sqrt(a * a + 1e-6)), rtol=1e-13, what="neg row")


def pin_expand_matches_matmul(o):
    """W^KV_b expand against a float64 matmul and the [K_h | V_h] column split."""
    g = torch.Generator().manual_seed(9)
    n, dl, hkv, dk = 21, 64, 3, 8
    c_hat = torch.randn(n, dl, generator=g, dtype=torch.float64)
    w = torch.randn(dl, hkv * 2 * dk, generator=g, dtype=torch.float32).to(torch.bfloat16)
    kv = (c_hat @ _f64(w)).reshape(n, hkv, 2 * dk)
    k, v = o.kv_expand(c_hat.numpy(), w, hkv, dk, dk)
    _close(k, kv[:, :, :dk].numpy(), rtol=1e-12, what="K")
    _close(v, kv[:, :, dk:].numpy(), rtol=1e-12, what="V")
    # one-hot W: latent coordinate l lands in head l // 16, slot l % 16
    eye = np.zeros((dl, hkv * 2 * dk))
    for l in range(min(dl, hkv * 2 * dk)):
        eye[l, l] = 1.0
    k1, v1 = o.kv_expand(c_hat.numpy(), eye, hkv, dk, dk)
    for l in range(hkv * 2 * dk):
        h, x = divmod(l, 2 * dk)
        val = (k1[:, h, x] if x < dk else v1[:, h, x - dk])
        _close(val, c_hat[:, l].numpy(), rtol=0, atol=0, what=f"one-hot col {l}")


# ---------------------------------------------------------------- identities

def pin_noise_equal_signal_cancels(o):
    """Q_noise[n] copied into every signal head of group n, lambda=1, G=1: O == 0."""
    for window, causal in ((0, True), (3, True), (0, False)):
        wl, x = _small(window=window, causal=causal)
        qs = x["q_noise"].repeat_interleave(wl.g, dim=2).contiguous()
        got = o.gdla_attn(qs, x["q_noise"], x["k"], x["v"], torch.ones_like(x["lam"]),
                          torch.ones_like(x["gate"]), window=window, causal=causal)
        assert np.all(got == 0.0), f"D=0 identity broken: max |O| = {np.abs(got).max()}"


def pin_window_covering_T_is_full(o):
    """A window of T or more keeps every causal key: identical to full causal."""
    wl, x = _small(T=17)
    full = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    for w in (wl.T, wl.T + 5):
        win = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], window=w)
        assert np.array_equal(full, win), f"window {w} differs from full causal"
    short = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                        window=wl.T - 1)
    assert not np.array_equal(full, short), "window T-1 must drop key 0 of the last row"


def pin_gate_is_elementwise(o):
    """gate=1 gives D itself; any gate G gives exactly G * D."""
    wl, x = _small()
    d_only = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"],
                         torch.ones_like(x["gate"]))
    gated = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    g = _f64(x["gate"]).reshape(wl.B * wl.T, -1).numpy()
    assert np.array_equal(gated, g * d_only), "O != G * D"
    assert not np.array_equal(gated, d_only)


def pin_linear_in_v(o):
    """O is linear in V for fixed Q, K, lambda, G."""
    wl, x = _small(seed=21)
    g = torch.Generator().manual_seed(22)
    v2 = torch.randn(x["v"].shape, generator=g, dtype=torch.float64)
    v1 = _f64(x["v"])
    args = (x["q_sig"], x["q_noise"], x["k"])
    o1 = o.gdla_attn(*args, v1, x["lam"], x["gate"])
    o2 = o.gdla_attn(*args, v2, x["lam"], x["gate"])
    o12 = o.gdla_attn(*args, v1 + 2.5 * v2, x["lam"], x["gate"])
    _close(o12, o1 + 2.5 * o2, rtol=1e-12, what="linearity in V")


def pin_key_shift_invariance(o):
    """Adding one vector to every key row of a KV head leaves softmax unchanged."""
    wl, x = _small(seed=31)
    g = torch.Generator().manual_seed(32)
    shift = torch.randn(1, 1, wl.Hkv, wl.d, generator=g, dtype=torch.float64)
    base = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    moved = o.gdla_attn(x["q_sig"], x["q_noise"], _f64(x["k"]) + shift, x["v"], x["lam"],
                        x["gate"])
    _close(moved, base, rtol=1e-10, what="key shift")


def pin_causality(o):
    """Changing keys/values after position i0 leaves rows <= i0 untouched."""
    wl, x = _small(seed=41)
    i0 = 9
    k2, v2 = x["k"].clone(), x["v"].clone()
    k2[:, i0 + 1:] = -k2[:, i0 + 1:] * 3
    v2[:, i0 + 1:] = v2[:, i0 + 1:] + 1
    a = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    b = o.gdla_attn(x["q_sig"], x["q_noise"], k2, v2, x["lam"], x["gate"])
    a = a.reshape(wl.B, wl.T, -1)
    b = b.reshape(wl.B, wl.T, -1)
    assert np.array_equal(a[:, :i0 + 1], b[:, :i0 + 1]), "future keys leaked into the past"
    assert not np.array_equal(a[:, i0 + 1:], b[:, i0 + 1:])


def pin_batch_permutation(o):
    """Permuting the batch permutes the output rows."""
    wl, x = _small(B=3, seed=51)
    perm = torch.tensor([2, 0, 1])
    a = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    xp = {k: v[perm] for k, v in x.items()}
    b = o.gdla_attn(xp["q_sig"], xp["q_noise"], xp["k"], xp["v"], xp["lam"], xp["gate"])
    assert np.array_equal(a.reshape(wl.B, wl.T, -1)[perm.numpy()], b.reshape(wl.B, wl.T, -1))


def pin_row_subset(o):
    """Evaluating a subset of rows gives exactly those rows of the full result."""
    wl, x = _small(seed=61)
    full = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    rows = [0, 5, wl.T - 1, wl.T, 2 * wl.T - 1]
    sub = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], rows=rows)
    assert np.array_equal(full[rows], sub)


def pin_row_gathered_inputs(o):
    """The row-gathered form equals the full form at those rows."""
    wl, x = _small(B=2, T=21, seed=65, window=6)
    rows = np.array([3, 0, 20, 21, 40, 33])
    full = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], window=6)
    flat = lambda t: t.reshape(wl.B * wl.T, *t.shape[2:])[torch.as_tensor(rows)]
    got = o.gdla_attn_rows(flat(x["q_sig"]), flat(x["q_noise"]), x["k"], x["v"], flat(x["lam"]),
                           flat(x["gate"]), rows, window=6)
    assert np.array_equal(full[rows], got)


def pin_scale_placement(o):
    """The scale multiplies q.k: doubling q and halving the scale changes nothing."""
    wl, x = _small(seed=71)
    sc = 1 / math.sqrt(wl.d)
    a = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], scale=sc)
    b = o.gdla_attn(_f64(x["q_sig"]) * 2, _f64(x["q_noise"]) * 2, x["k"], x["v"], x["lam"],
                    x["gate"], scale=sc / 2)
    assert np.array_equal(a, b)
    c = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    assert np.array_equal(a, c), "default scale must be 1/sqrt(d)"


# ---------------------------------------------------------------- rotary term
# "Motif 3: Technical Report" (paper.rainbus.top digest), "technical novelty"
# paragraph: both query paths share the up-projected KV and one broadcast
# decoupled rotary key.  Reading: score = scale * (q.k + q_r.k_r), one rotary
# key per token for every head of both paths; default scale 1/sqrt(d + d_rope).

def _golden_value(x):
    if isinstance(x, str):
        if x in ("LN2", "LN3"):
            return math.log(2.0 if x == "LN2" else 3.0)
        num, den = x.split("/")
        return float(num) / float(den)
    return x


def _golden_array(a):
    if isinstance(a, list):
        return [_golden_array(e) for e in a]
    return _golden_value(a)


def _rope_small(B=2, T=19, Hs=8, Hn=2, Hkv=2, d=16, dr=8, seed=3, window=0, causal=True):
    wl, x = _small(B, T, Hs, Hn, Hkv, d, seed=seed, window=window, causal=causal)
    g = torch.Generator().manual_seed(seed + 1000)
    x["q_rope_sig"] = torch.randn(B, T, Hs, dr, generator=g).to(torch.bfloat16)
    x["q_rope_noise"] = torch.randn(B, T, Hn, dr, generator=g).to(torch.bfloat16)
    x["k_rope"] = torch.randn(B, T, dr, generator=g).to(torch.bfloat16)
    return wl, x


def _rope_attn(o, x, **kw):
    return o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                       q_rope_sig=x["q_rope_sig"], q_rope_noise=x["q_rope_noise"],
                       k_rope=x["k_rope"], **kw)


def pin_rope_hand_example(o):
    """Two-token case with the rotary term, derived by hand
    (tests/golden/rope_hand_example.json)."""
    with open(os.path.join(GOLDEN, "rope_hand_example.json")) as f:
        g = json.load(f)
    arr = lambda key: np.array(_golden_array(g[key]), dtype=np.float64)
    args = dict(q_sig=arr("q_sig"), q_noise=arr("q_noise"), k=arr("k"), v=arr("v"),
                lam=arr("lam"), gate=arr("gate"), q_rope_sig=arr("q_rope_sig"),
                q_rope_noise=arr("q_rope_noise"), k_rope=arr("k_rope"),
                scale=g["shape"]["scale"])
    exp = {k: np.array(_golden_array(v)) for k, v in g["expected"].items()}
    _close(o.gdla_attn(**args, window=0, causal=True), exp["causal"], what="rope causal")
    _close(o.gdla_attn(**args, window=1, causal=True), exp["window1"], what="rope W=1")
    _close(o.gdla_attn(**args, window=0, causal=False), exp["noncausal"],
           what="rope non-causal")


def pin_rope_matches_sdpa_on_concatenated_heads(o):
    """torch SDPA on [q | q_r] against [k_h | k_r] (the one rotary key
    concatenated to every KV head), then the differential and gate."""
    for window, causal in ((0, True), (5, True), (0, False)):
        wl, x = _rope_small(seed=41 + window, window=window, causal=causal)
        dr = x["k_rope"].shape[-1]
        sc = 1.0 / math.sqrt(wl.d + dr)
        kr = _f64(x["k_rope"]).unsqueeze(2).expand(-1, -1, wl.Hkv, -1)
        kcat = torch.cat([_f64(x["k"]), kr], dim=-1)
        # SDPA takes a value width (d) other than the key width (d + d_rope)
        hs = _sdpa(torch.cat([_f64(x["q_sig"]), _f64(x["q_rope_sig"])], -1), kcat, x["v"],
                   wl.Hs // wl.Hkv, window, causal, sc)
        hn = _sdpa(torch.cat([_f64(x["q_noise"]), _f64(x["q_rope_noise"])], -1), kcat, x["v"],
                   1, window, causal, sc)
        g = wl.Hs // wl.Hn
        dd = hs - _f64(x["lam"]).unsqueeze(-1) * hn.repeat_interleave(g, dim=2)
        want = (_f64(x["gate"]).view(wl.B, wl.T, wl.Hs, wl.d) * dd).reshape(wl.B * wl.T, -1)
        _close(_rope_attn(o, x, window=window, causal=causal), want.numpy(), rtol=1e-10,
               atol=1e-12, what=f"rope vs SDPA (window {window}, causal {causal})")


def pin_rope_zero_terms_leave_plain_scores(o):
    """Zero rotary queries and keys add nothing: with the same scale the
    result equals the oracle without the rotary term, bit for bit."""
    wl, x = _rope_small(seed=43)
    sc = 1.0 / math.sqrt(wl.d)
    plain = o.gdla_attn(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"], scale=sc)
    for name in ("q_rope_sig", "q_rope_noise", "k_rope"):
        x[name] = torch.zeros_like(x[name])
    assert np.array_equal(_rope_attn(o, x, scale=sc), plain)


def pin_rope_key_shift_invariance(o):
    """Adding one vector c to every rotary key adds q_r.c to every score of a
    row (per head), which the softmax removes: O is unchanged."""
    wl, x = _rope_small(seed=44, window=4)
    a = _rope_attn(o, x, window=4)
    x["k_rope"] = _f64(x["k_rope"]) + torch.linspace(-2, 3, x["k_rope"].shape[-1],
                                                     dtype=torch.float64)
    _close(_rope_attn(o, x, window=4), a, rtol=1e-9, atol=1e-12, what="rope shift")


def pin_rope_key_is_per_token_not_per_query(o):
    """Row i's rotary scores use key j's rotary vector: changing the rotary
    key of one earlier token changes row i, changing a later one does not."""
    wl, x = _rope_small(B=1, seed=45)
    a = _rope_attn(o, x)
    kr = x["k_rope"].clone()
    kr[0, 3] += 2.0
    x2 = dict(x, k_rope=kr)
    b = _rope_attn(o, x2)
    assert np.array_equal(a[:3], b[:3]), "rows before the changed key must not move"
    assert not np.allclose(a[10], b[10]), "a later row must see the changed rotary key"


def pin_rope_default_scale(o):
    """The default scale with the rotary term is 1/sqrt(d + d_rope)."""
    wl, x = _rope_small(seed=46)
    dr = x["k_rope"].shape[-1]
    assert np.array_equal(_rope_attn(o, x), _rope_attn(o, x, scale=1 / math.sqrt(wl.d + dr)))


def pin_rope_rows_match_full(o):
    wl, x = _rope_small(seed=47, window=6)
    rows = np.array([3, 0, 20, 21, 37, 33])
    full = _rope_attn(o, x, window=6)
    flat = lambda t: t.reshape(wl.B * wl.T, *t.shape[2:])[torch.as_tensor(rows)]
    got = o.gdla_attn_rows(flat(x["q_sig"]), flat(x["q_noise"]), x["k"], x["v"], flat(x["lam"]),
                           flat(x["gate"]), rows, window=6, q_rope_sig_rows=flat(x["q_rope_sig"]),
                           q_rope_noise_rows=flat(x["q_rope_noise"]), k_rope=x["k_rope"])
    assert np.array_equal(full[rows], got)


# ---------------------------------------------------------------- decode
# The decode reads the KV latent cache ("Motif 3: Technical Report",
# paper.rainbus.top, "technical novelty" paragraph: the inference cache is the
# latent, the size of MLA's) and computes the forward pass for each
# sequence's newest token.


def _decode_case(B=3, L_max=37, Hs=8, Hn=2, d=16, dl=64, seed=5):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *shape, s=1.0: (torch.randn(*shape, generator=g) * s).to(torch.bfloat16)
    x = {
        "q_sig": bf(B, Hs, d), "q_noise": bf(B, Hn, d), "c_kv": bf(B, L_max, dl),
        "w_kvb": bf(dl, Hn * 2 * d, s=dl ** -0.5),
        "lam": torch.sigmoid(torch.randn(B, Hs, generator=g)).to(torch.bfloat16),
        "gate": torch.sigmoid(torch.randn(B, Hs * d, generator=g)).to(torch.bfloat16),
        "rms_w": (torch.rand(dl, generator=g) + 0.5).to(torch.bfloat16),
    }
    return x, (B, L_max, Hs, Hn, d, dl)


def _decode_torch(x, lens, window, eps=1e-6, use_w=True):
    """The decode by torch library routines in float64: rms_norm, matmul,
    SDPA for the one query row, then the differential combine and gate."""
    B, Hs, d = x["q_sig"].shape
    Hn = x["q_noise"].shape[1]
    g = Hs // Hn
    w = _f64(x["w_kvb"])
    out = []
    for b in range(B):
        L = int(lens[b])
        c = _f64(x["c_kv"][b, :L])
        chat = F.rms_norm(c, (c.shape[-1],), weight=_f64(x["rms_w"]) if use_w else None, eps=eps)
        kv = (chat @ w).view(L, Hn, 2 * d)
        k, v = kv[..., :d], kv[..., d:]
        lo = max(0, L - window) if window > 0 else 0

        def attend(q, heads_per_kv):  # q [H, d] -> [H, d]
            kk = k[lo:].repeat_interleave(heads_per_kv, dim=1).permute(1, 0, 2)
            vv = v[lo:].repeat_interleave(heads_per_kv, dim=1).permute(1, 0, 2)
            return F.scaled_dot_product_attention(q.unsqueeze(1), kk, vv,
                                                  scale=1.0 / math.sqrt(d)).squeeze(1)
        hs = attend(_f64(x["q_sig"][b]), g)
        hn = attend(_f64(x["q_noise"][b]), 1)
        dd = hs - _f64(x["lam"][b]).unsqueeze(1) * hn.repeat_interleave(g, dim=0)
        out.append((_f64(x["gate"][b]).view(Hs, d) * dd).reshape(-1))
    return torch.stack(out).numpy()


def pin_decode_matches_torch_expand_sdpa(o):
    x, (B, L_max, Hs, Hn, d, dl) = _decode_case()
    lens = [37, 1, 20]
    for window in (0, 5):
        got = o.decode(x["q_sig"], x["q_noise"], x["c_kv"], lens, x["w_kvb"], x["lam"],
                       x["gate"], rms_w=x["rms_w"], window=window)
        _close(got, _decode_torch(x, lens, window), rtol=1e-10, atol=1e-12,
               what=f"decode vs torch (window {window})")


def pin_decode_rope_matches_torch(o):
    """Decode with the rotary term: the cache holds each token's rotary key
    beside its latent (as MLA caches it); torch float64 rms_norm, matmul and
    SDPA on the concatenated [q | q_r] / [k_h | k_r] give the same row."""
    x, (B, L_max, Hs, Hn, d, dl) = _decode_case(seed=12)
    dr = 8
    g_ = torch.Generator().manual_seed(99)
    qrs = torch.randn(B, Hs, dr, generator=g_).to(torch.bfloat16)
    qrn = torch.randn(B, Hn, dr, generator=g_).to(torch.bfloat16)
    kr = torch.randn(B, L_max, dr, generator=g_).to(torch.bfloat16)
    g = Hs // Hn
    w = _f64(x["w_kvb"])
    for window, lens in ((0, [37, 1, 20]), (5, [37, 4, 20])):
        got = o.decode(x["q_sig"], x["q_noise"], x["c_kv"], lens, x["w_kvb"], x["lam"],
                       x["gate"], rms_w=x["rms_w"], window=window, q_rope_sig=qrs,
                       q_rope_noise=qrn, k_rope=kr)
        for b in range(B):
            L = lens[b]
            c = _f64(x["c_kv"][b, :L])
            chat = F.rms_norm(c, (dl,), weight=_f64(x["rms_w"]), eps=1e-6)
            kv = (chat @ w).view(L, Hn, 2 * d)
            lo = max(0, L - window) if window > 0 else 0
            k = torch.cat([kv[lo:, :, :d], _f64(kr[b, lo:L]).unsqueeze(1).expand(-1, Hn, -1)], -1)
            v = kv[lo:, :, d:]

            def attend(q, qr, rep):
                kk = k.repeat_interleave(rep, dim=1).permute(1, 0, 2)
                vv = v.repeat_interleave(rep, dim=1).permute(1, 0, 2)
                qq = torch.cat([_f64(q), _f64(qr)], -1).unsqueeze(1)
                return F.scaled_dot_product_attention(qq, kk, vv,
                                                      scale=1 / math.sqrt(d + dr)).squeeze(1)
            hs = attend(x["q_sig"][b], qrs[b], g)
            hn = attend(x["q_noise"][b], qrn[b], 1)
            dd = hs - _f64(x["lam"][b]).unsqueeze(1) * hn.repeat_interleave(g, dim=0)
            want = (_f64(x["gate"][b]).view(Hs, d) * dd).reshape(-1).numpy()
            _close(got[b], want, rtol=1e-10, atol=1e-12, what=f"rope decode W={window} b={b}")


def pin_decode_absorbed_latent_form(o):
    """W^KV_b absorbed into the query and the output: scores q.(c_hat W_K)
    = (W_K q).c_hat and sum_j p_j (c_hat_j W_V) = (sum_j p_j c_hat_j) W_V,
    so the decode can run in the 512-d latent space.  Written out here in
    numpy, it must equal the oracle's expand-then-attend decode."""
    x, (B, L_max, Hs, Hn, d, dl) = _decode_case(seed=8)
    lens = [30, 37, 2]
    got = o.decode(x["q_sig"], x["q_noise"], x["c_kv"], lens, x["w_kvb"], x["lam"], x["gate"],
                   rms_w=x["rms_w"])
    W = x["w_kvb"].double().numpy().reshape(dl, Hn, 2 * d)
    g = Hs // Hn
    rw = x["rms_w"].double().numpy()
    for b in range(B):
        L = lens[b]
        c = x["c_kv"][b, :L].double().numpy()
        chat = c / np.sqrt((c * c).mean(axis=1, keepdims=True) + 1e-6) * rw

        def latent_head(q, kvh):
            qt = W[:, kvh, :d] @ q                 # absorbed query, [dl]
            s = chat @ qt / math.sqrt(d)
            p = np.exp(s - s.max())
            z = p @ chat / p.sum()                 # attention in latent space, [dl]
            return z @ W[:, kvh, d:]               # absorbed output projection
        hn = [latent_head(x["q_noise"][b, n].double().numpy(), n) for n in range(Hn)]
        for h in range(Hs):
            hs = latent_head(x["q_sig"][b, h].double().numpy(), h // g)
            want = x["gate"][b, h * d:(h + 1) * d].double().numpy() * (
                hs - float(x["lam"][b, h]) * hn[h // g])
            _close(got[b, h * d:(h + 1) * d], want, rtol=1e-10, atol=1e-12,
                   what=f"absorbed decode b={b} h={h}")


def pin_decode_single_token_and_window_one(o):
    """One cached token, or a window of 1: O = G (.) (1 - lambda) V_last with
    V_last = RMSNorm(c_last) W_V of the head's KV group."""
    x, (B, L_max, Hs, Hn, d, dl) = _decode_case(seed=9)
    g = Hs // Hn
    W = x["w_kvb"].double().numpy().reshape(dl, Hn, 2 * d)
    rw = x["rms_w"].double().numpy()
    for lens, window in (([1, 1, 1], 0), ([37, 12, 3], 1)):
        got = o.decode(x["q_sig"], x["q_noise"], x["c_kv"], lens, x["w_kvb"], x["lam"],
                       x["gate"], rms_w=x["rms_w"], window=window)
        for b in range(B):
            c = x["c_kv"][b, lens[b] - 1].double().numpy()
            chat = c / np.sqrt((c * c).mean() + 1e-6) * rw
            for h in range(Hs):
                v = chat @ W[:, h // g, d:]
                want = x["gate"][b, h * d:(h + 1) * d].double().numpy() * \
                    (1.0 - float(x["lam"][b, h])) * v
                _close(got[b, h * d:(h + 1) * d], want, rtol=1e-12, atol=1e-13,
                       what=f"decode closed form lens={lens} b={b} h={h}")


def pin_decode_ignores_rows_past_the_length(o):
    x, _ = _decode_case(seed=10)
    lens = [10, 37, 25]
    a = o.decode(x["q_sig"], x["q_noise"], x["c_kv"], lens, x["w_kvb"], x["lam"], x["gate"])
    c2 = x["c_kv"].clone()
    for b, L in enumerate(lens):
        c2[b, L:] = 1e3
    bb = o.decode(x["q_sig"], x["q_noise"], c2, lens, x["w_kvb"], x["lam"], x["gate"])
    assert np.array_equal(a, bb), "decode read cache rows past the sequence length"
    c2[1, 36] += 1.0  # the query token's own latent does count
    cc = o.decode(x["q_sig"], x["q_noise"], c2, lens, x["w_kvb"], x["lam"], x["gate"])
    assert not np.array_equal(a[1], cc[1])


# ---------------------------------------------------------------- backward
# The model is trained with GDLA ("Вышла новая модель Motif 3", pikabu.ru);
# the backward is the gradient of the forward of [R] step 2.


def _bwd_case(B=1, T=6, Hs=4, Hn=2, Hkv=2, d=3, seed=21):
    g = torch.Generator().manual_seed(seed)
    f = lambda *shape: torch.randn(*shape, generator=g, dtype=torch.float64)
    x = {"q_sig": f(B, T, Hs, d), "q_noise": f(B, T, Hn, d), "k": f(B, T, Hkv, d),
         "v": f(B, T, Hkv, d),
         "lam": torch.sigmoid(f(B, T, Hs)), "gate": torch.sigmoid(f(B, T, Hs * d))}
    return x, f(B, T, Hs * d)


def pin_bwd_finite_differences(o):
    """Every gradient element against central differences of the (pinned)
    forward oracle: d/dtheta sum(dO * O) ~ (L(theta + e) - L(theta - e)) / 2e."""
    for window, causal in ((0, True), (2, True), (0, False)):
        x, dout = _bwd_case(seed=21 + window + 5 * int(causal))
        grads = o.gdla_attn_bwd(*(x[n] for n in ("q_sig", "q_noise", "k", "v", "lam", "gate")),
                                dout, window=window, causal=causal, scale=0.7)
        loss = lambda xx: float((o.gdla_attn(xx["q_sig"], xx["q_noise"], xx["k"], xx["v"],
                                              xx["lam"], xx["gate"], window=window,
                                              causal=causal, scale=0.7)
                                 * dout.reshape(-1, dout.shape[-1]).numpy()).sum())
        eps = 1e-6
        for name, gname in (("q_sig", "dq_sig"), ("q_noise", "dq_noise"), ("k", "dk"),
                            ("v", "dv"), ("lam", "dlam"), ("gate", "dgate")):
            t = x[name]
            num = np.empty(t.numel())
            flat = t.view(-1)
            for idx in range(t.numel()):
                keep = float(flat[idx])
                flat[idx] = keep + eps
                lp = loss(x)
                flat[idx] = keep - eps
                lm = loss(x)
                flat[idx] = keep
                num[idx] = (lp - lm) / (2 * eps)
            _close(grads[gname].reshape(-1), num, rtol=1e-6, atol=1e-7,
                   what=f"{gname} vs finite differences (window {window}, causal {causal})")


def pin_bwd_matches_torch_autograd(o):
    """torch float64 autograd through SDPA (KV heads repeated per group), the
    differential and the gate."""
    for window, causal in ((0, True), (5, True), (0, False)):
        wl, x = _small(seed=77 + window, window=window, causal=causal)
        g = torch.Generator().manual_seed(5)
        dout = torch.randn(wl.B, wl.T, wl.Hs * wl.d, generator=g, dtype=torch.float64)
        leaves = {n: _f64(x[n]).clone().requires_grad_(True)
                  for n in ("q_sig", "q_noise", "k", "v", "lam", "gate")}
        sc = 1.0 / math.sqrt(wl.d)
        hs = _sdpa(leaves["q_sig"], leaves["k"], leaves["v"], wl.Hs // wl.Hkv, window, causal, sc)
        hn = _sdpa(leaves["q_noise"], leaves["k"], leaves["v"], 1, window, causal, sc)
        dd = hs - leaves["lam"].unsqueeze(-1) * hn.repeat_interleave(wl.g, dim=2)
        out = (leaves["gate"].view(wl.B, wl.T, wl.Hs, wl.d) * dd).reshape(wl.B, wl.T, -1)
        (out * dout).sum().backward()
        got = o.gdla_attn_bwd(*(x[n] for n in ("q_sig", "q_noise", "k", "v", "lam", "gate")),
                              dout, window=window, causal=causal)
        for name, gname in (("q_sig", "dq_sig"), ("q_noise", "dq_noise"), ("k", "dk"),
                            ("v", "dv"), ("lam", "dlam"), ("gate", "dgate")):
            _close(got[gname], leaves[name].grad.numpy(), rtol=1e-10, atol=1e-12,
                   what=f"{gname} vs torch autograd (window {window}, causal {causal})")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
