"""Float64 CPU oracle for the GDLA forward pass (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library never loads
it, and it imports nothing from the product package: the two share no code.

The arithmetic lives in ``gdla_oracle.c`` (plain C, double precision, OpenMP
over rows and heads); this module only compiles it with gcc and marshals
arrays.  Inputs may be CPU torch tensors (bfloat16, float32, float64) or numpy
arrays (float32, float64, or uint16 holding bfloat16 bits); bfloat16 is handed
to C as raw bit patterns and widened there exactly.  Results are float64 numpy
arrays.

Each function restates one step of the forward pass as the page
"Motif 3: Technical Report" (paper.rainbus.top digest), step 2 "GDLA forward",
writes it; ``gdla_oracle.c`` lists the readings taken where the page is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gdla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle_gdla.so")

BF16, F64, F32 = 0, 1, 2


def compile_source(src: str, out: str) -> str:
    """Compile one oracle C source into a shared library (gcc, OpenMP)."""
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``gdla_oracle.c`` into ``oracle/_liboracle_gdla.so`` if stale."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(SOURCE)):
        return _LIB_PATH
    return compile_source(SOURCE, _LIB_PATH)


def _arr(x):
    """Return (contiguous host array, pointer, dtype code) for one input."""
    import torch
    if isinstance(x, torch.Tensor):
        x = x.detach()
        if x.device.type != "cpu":
            raise ValueError("oracle inputs must live on the CPU")
        x = x.contiguous()
        if x.dtype == torch.bfloat16:
            a = x.view(torch.int16).numpy().view(np.uint16)
            return a, a.ctypes.data, BF16
        if x.dtype == torch.float32:
            a = x.numpy()
            return a, a.ctypes.data, F32
        a = x.to(torch.float64).numpy()
        return a, a.ctypes.data, F64
    a = np.ascontiguousarray(x)
    if a.dtype == np.float32:
        return a, a.ctypes.data, F32
    if a.dtype == np.uint16:  # raw bfloat16 bits
        return a, a.ctypes.data, BF16
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data, F64


def _rows(rows, total):
    if rows is None:
        return None, None, total
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    if r.size and (r.min() < 0 or r.max() >= total):
        raise ValueError("row index out of range")
    return r, r.ctypes.data, int(r.size)


class Oracle:
    """Bindings to one compiled copy of the C oracle."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.gdla_oracle_rmsnorm.argtypes = [vp, i32, vp, i32, f64, i64, i32, vp]
        lib.gdla_oracle_rmsnorm.restype = None
        lib.gdla_oracle_kv_expand.argtypes = [vp, vp, i32, i64, i32, i32, i32, i32, vp, vp]
        lib.gdla_oracle_kv_expand.restype = None
        lib.gdla_oracle_attention_path.argtypes = [vp, i32, vp, i32, vp, i32, i32, i64, i32, i32,
                                                   i32, i64, i32, f64, vp, i64, vp]
        lib.gdla_oracle_attention_path.restype = None
        lib.gdla_oracle_differential_gate.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32,
                                                      vp, i64, vp]
        lib.gdla_oracle_differential_gate.restype = None
        lib.gdla_oracle_attn.argtypes = [vp, i32, vp, i32, vp, i32, vp, i32, vp, i32, vp, i32,
                                         i32, i64, i32, i32, i32, i32, i64, i32, f64, vp, i64, vp]
        lib.gdla_oracle_attn.restype = ctypes.c_int
        lib.gdla_oracle_attn_compact.argtypes = [vp, i32, vp, i32, vp, i32, vp, i32, vp, i32, vp,
                                                 i32, i64, i32, i32, i32, i32, i64, i32, f64, vp,
                                                 i64, vp]
        lib.gdla_oracle_attn_compact.restype = ctypes.c_int
        lib.gdla_oracle_attn_rope.argtypes = [vp, i32, vp, i32, vp, i32, vp, i32, vp, i32, vp,
                                              i32, i32, vp, i32, vp, i32, vp, i32, i32, i64, i32,
                                              i32, i32, i32, i64, i32, f64, vp, i64, vp]
        lib.gdla_oracle_attn_rope.restype = ctypes.c_int
        lib.gdla_oracle_decode.argtypes = [vp, i32, vp, i32, vp, i32, vp, i32, vp, i32, vp, i32,
                                           i32, vp, vp, i32, f64, vp, i32, vp, i32, vp, i32, i32,
                                           i64, i32, i32, i32, i32, i32, i64, f64, vp]
        lib.gdla_oracle_decode.restype = ctypes.c_int
        lib.gdla_oracle_attn_bwd.argtypes = [vp, i32, vp, i32, vp, i32, vp, i32, vp, i32, vp, i32,
                                             vp, i32, i32, i64, i32, i32, i32, i32, i64, i32, f64,
                                             vp, vp, vp, vp, vp, vp]
        lib.gdla_oracle_attn_bwd.restype = ctypes.c_int
        lib.gdla_oracle_version.restype = ctypes.c_int
        self.lib = lib
        self.path = lib_path

    # a1: RMSNorm of the KV latent
    def rmsnorm(self, c, w=None, eps: float = 1e-6) -> np.ndarray:
        """c / sqrt(mean(c^2) + eps) * w, row by row; w=None means ones."""
        ca, cp, cdt = _arr(c)
        n, dl = ca.shape[0], ca.shape[-1]
        out = np.empty((n, dl), dtype=np.float64)
        wa, wp, wdt = (None, None, F64) if w is None else _arr(w)
        self.lib.gdla_oracle_rmsnorm(cp, cdt, wp, wdt, float(eps), n, dl, out.ctypes.data)
        return out

    # a2: W^KV_b up-projection
    def kv_expand(self, c_hat, w_kvb, n_kv_heads: int, dk: int, dv: int):
        """Returns K [N,Hkv,dk], V [N,Hkv,dv] from the normalised latent."""
        ch = np.ascontiguousarray(np.asarray(c_hat, dtype=np.float64))
        wa, wp, wdt = _arr(w_kvb)
        n, dl = ch.shape
        if tuple(wa.shape) != (dl, n_kv_heads * (dk + dv)):
            raise ValueError("W^KV_b must be [d_latent, Hkv*(dk+dv)]")
        k = np.empty((n, n_kv_heads, dk), dtype=np.float64)
        v = np.empty((n, n_kv_heads, dv), dtype=np.float64)
        self.lib.gdla_oracle_kv_expand(ch.ctypes.data, wp, wdt, n, dl, n_kv_heads, dk, dv,
                                       k.ctypes.data, v.ctypes.data)
        return k, v

    # a3/a4/a5: one attention path under the mask
    def attention_path(self, q, k, v, window: int = 0, causal: bool = True, scale=None,
                       rows=None) -> np.ndarray:
        """q [B,T,H,d], k/v [B,T,Hkv,d]; head h reads KV head h // (H // Hkv).

        Returns H[n_rows, H, d] for flat rows b*T+i (every row when None).
        """
        qa, qp, qdt = _arr(q)
        ka, kp, kdt = _arr(k)
        va, vp, vdt = _arr(v)
        B, T, H, d = qa.shape
        Hkv = ka.shape[2]
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        r, rp, n = _rows(rows, B * T)
        out = np.empty((n, H, d), dtype=np.float64)
        self.lib.gdla_oracle_attention_path(qp, qdt, kp, kdt, vp, vdt, B, T, H, Hkv, d,
                                            int(window), int(bool(causal)), float(scale), rp, n,
                                            out.ctypes.data)
        return out

    # a6/a7/a8: Repeat_g, differential combine, gate
    def differential_gate(self, hs, hn, lam, gate, rows=None) -> np.ndarray:
        """D = H_S - lambda * Repeat_g(H_N); O = G * D.  Returns O[n_rows, Hs*d].

        hs [n,Hs,d] and hn [n,Hn,d] are per evaluated row; lam [..,Hs] and
        gate [..,Hs*d] are addressed by the flat row index (rows, or 0..n-1).
        """
        hs = np.ascontiguousarray(np.asarray(hs, dtype=np.float64))
        hn = np.ascontiguousarray(np.asarray(hn, dtype=np.float64))
        la, lp, ldt = _arr(lam)
        ga, gp, gdt = _arr(gate)
        n, Hs, d = hs.shape
        Hn = hn.shape[1]
        r, rp, nr = _rows(rows, la.size // Hs)
        if rows is not None and nr != n:
            raise ValueError("rows must list one flat index per evaluated row")
        out = np.empty((n, Hs * d), dtype=np.float64)
        self.lib.gdla_oracle_differential_gate(hs.ctypes.data, hn.ctypes.data, lp, ldt, gp, gdt,
                                               Hs, Hn, d, rp, n, out.ctypes.data)
        return out

    # whole attention forward
    def gdla_attn(self, q_sig, q_noise, k, v, lam, gate, window: int = 0, causal: bool = True,
                  scale=None, rows=None, q_rope_sig=None, q_rope_noise=None,
                  k_rope=None) -> np.ndarray:
        """O[n_rows, Hs*d] in float64 for flat rows b*T+i (all when None).

        q_sig [B,T,Hs,d], q_noise [B,T,Hn,d], k/v [B,T,Hkv,d], lam [B,T,Hs],
        gate [B,T,Hs*d].  With the decoupled rotary term: q_rope_sig
        [B,T,Hs,dr], q_rope_noise [B,T,Hn,dr] and k_rope [B,T,dr] (one rotary
        key per token for every head); the default scale is then
        1/sqrt(d + dr).
        """
        if k_rope is not None:
            return self._attn_rope(q_sig, q_noise, q_rope_sig, q_rope_noise, k, k_rope, v, lam,
                                   gate, window, causal, scale, rows, compact=False)
        qs, qsp, qsdt = _arr(q_sig)
        qn, qnp, qndt = _arr(q_noise)
        ka, kp, kdt = _arr(k)
        va, vp, vdt = _arr(v)
        la, lp, ldt = _arr(lam)
        ga, gp, gdt = _arr(gate)
        B, T, Hs, d = qs.shape
        Hn = qn.shape[2]
        Hkv = ka.shape[2]
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        r, rp, n = _rows(rows, B * T)
        out = np.empty((n, Hs * d), dtype=np.float64)
        rc = self.lib.gdla_oracle_attn(qsp, qsdt, qnp, qndt, kp, kdt, vp, vdt, lp, ldt, gp, gdt,
                                       B, T, Hs, Hn, Hkv, d, int(window), int(bool(causal)),
                                       float(scale), rp, n, out.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected the head counts (need Hs % Hn == 0, Hn == Hkv)")
        return out


    def _attn_rope(self, q_sig, q_noise, qr_sig, qr_noise, k, k_rope, v, lam, gate, window,
                   causal, scale, rows, compact):
        qs, qsp, qsdt = _arr(q_sig)
        qn, qnp, qndt = _arr(q_noise)
        rs, rsp, rsdt = _arr(qr_sig)
        rn, rnp, rndt = _arr(qr_noise)
        ka, kp, kdt = _arr(k)
        kr, krp, krdt = _arr(k_rope)
        va, vp, vdt = _arr(v)
        la, lp, ldt = _arr(lam)
        ga, gp, gdt = _arr(gate)
        B, T, Hkv, d = ka.shape
        dr = kr.shape[-1]
        Hs, Hn = qs.shape[-2], qn.shape[-2]
        if tuple(kr.shape) != (B, T, dr) or rs.shape[-1] != dr or rn.shape[-1] != dr:
            raise ValueError("k_rope must be [B,T,dr] and the rotary queries [..., H, dr]")
        if rs.shape[:-1] != qs.shape[:-1] or rn.shape[:-1] != qn.shape[:-1]:
            raise ValueError("rotary queries must be laid out like the queries")
        if scale is None:
            scale = 1.0 / np.sqrt(d + dr)
        r, rp, n = _rows(rows, B * T)
        if compact and (qs.shape[0] != n or la.shape[0] != n or ga.shape[0] != n):
            raise ValueError("row-gathered inputs must have one entry per row")
        out = np.empty((n, Hs * d), dtype=np.float64)
        rc = self.lib.gdla_oracle_attn_rope(qsp, qsdt, qnp, qndt, rsp, rsdt, rnp, rndt, kp, kdt,
                                            krp, krdt, dr, vp, vdt, lp, ldt, gp, gdt,
                                            int(bool(compact)), T, Hs, Hn, Hkv, d, int(window),
                                            int(bool(causal)), float(scale), rp, n,
                                            out.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected the head counts or the rotary inputs")
        return out

    def gdla_attn_rows(self, q_sig_rows, q_noise_rows, k, v, lam_rows, gate_rows, rows,
                       window: int = 0, causal: bool = True, scale=None, q_rope_sig_rows=None,
                       q_rope_noise_rows=None, k_rope=None) -> np.ndarray:
        """Same as gdla_attn, with the query-side inputs gathered per row.

        q_sig_rows [n,Hs,d], q_noise_rows [n,Hn,d], lam_rows [n,Hs] and
        gate_rows [n,Hs*d] hold only the evaluated rows (flat indices b*T+i in
        ``rows``, same order); k and v stay full [B,T,Hkv,d].  With the
        rotary term, q_rope_*_rows [n,H,dr] are gathered too and k_rope
        [B,T,dr] stays full.
        """
        if k_rope is not None:
            return self._attn_rope(q_sig_rows, q_noise_rows, q_rope_sig_rows, q_rope_noise_rows,
                                   k, k_rope, v, lam_rows, gate_rows, window, causal, scale,
                                   rows, compact=True)
        qs, qsp, qsdt = _arr(q_sig_rows)
        qn, qnp, qndt = _arr(q_noise_rows)
        ka, kp, kdt = _arr(k)
        va, vp, vdt = _arr(v)
        la, lp, ldt = _arr(lam_rows)
        ga, gp, gdt = _arr(gate_rows)
        B, T, Hkv, d = ka.shape
        n, Hs = qs.shape[0], qs.shape[1]
        Hn = qn.shape[1]
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        r, rp, nr = _rows(rows, B * T)
        if nr != n or la.shape[0] != n or ga.shape[0] != n:
            raise ValueError("row-gathered inputs must have one entry per row")
        out = np.empty((n, Hs * d), dtype=np.float64)
        rc = self.lib.gdla_oracle_attn_compact(qsp, qsdt, qnp, qndt, kp, kdt, vp, vdt, lp, ldt, gp,
                                               gdt, T, Hs, Hn, Hkv, d, int(window),
                                               int(bool(causal)), float(scale), rp, n,
                                               out.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected the head counts (need Hs % Hn == 0, Hn == Hkv)")
        return out


    # decode: the newest token of each sequence over its latent cache
    def decode(self, q_sig, q_noise, c_kv, cache_len, w_kvb, lam, gate, rms_w=None,
               eps: float = 1e-6, window: int = 0, scale=None, q_rope_sig=None,
               q_rope_noise=None, k_rope=None) -> np.ndarray:
        """O[B, Hs*d] for the query token of each sequence (its position is
        cache_len[b] - 1), from the raw KV latents c_kv [B, L_max, d_latent]:
        RMSNorm, W^KV_b expand, then the GDLA forward for that one row.

        q_sig [B,Hs,d], q_noise [B,Hn,d], lam [B,Hs], gate [B,Hs*d];
        cache_len: B integers in 1..L_max.  With the rotary term: the cached
        rotary keys k_rope [B,L_max,dr] and the query token's q_rope_sig
        [B,Hs,dr], q_rope_noise [B,Hn,dr]; the default scale is then
        1/sqrt(d + dr).
        """
        qs, qsp, qsdt = _arr(q_sig)
        qn, qnp, qndt = _arr(q_noise)
        dr = 0
        rsp = rnp = krp = None
        rsdt = rndt = krdt = F64
        if k_rope is not None:
            rs, rsp, rsdt = _arr(q_rope_sig)
            rn, rnp, rndt = _arr(q_rope_noise)
            kr, krp, krdt = _arr(k_rope)
            dr = kr.shape[-1]
            if rs.shape != (qs.shape[0], qs.shape[1], dr) or \
                    rn.shape != (qn.shape[0], qn.shape[1], dr):
                raise ValueError("rotary queries must be [B, H, dr]")
        ca, cp, cdt = _arr(c_kv)
        wa, wp, wdt = _arr(w_kvb)
        la, lp, ldt = _arr(lam)
        ga, gp, gdt = _arr(gate)
        ra, rp, rdt = (None, None, F64) if rms_w is None else _arr(rms_w)
        B, Hs, d = qs.shape
        Hn = qn.shape[1]
        L_max, dl = ca.shape[1], ca.shape[2]
        Hkv = wa.shape[1] // (2 * d)
        lens = np.ascontiguousarray(np.asarray(cache_len, dtype=np.int64).reshape(-1))
        if lens.size != B or lens.min() < 1 or lens.max() > L_max:
            raise ValueError("cache_len must hold B lengths in 1..L_max")
        if dr and tuple(kr.shape) != (B, L_max, dr):
            raise ValueError("k_rope must be [B, L_max, dr]")
        if scale is None:
            scale = 1.0 / np.sqrt(d + dr)
        out = np.empty((B, Hs * d), dtype=np.float64)
        rc = self.lib.gdla_oracle_decode(qsp, qsdt, qnp, qndt, rsp, rsdt, rnp, rndt, cp, cdt, krp,
                                         krdt, dr, lens.ctypes.data, rp, rdt, float(eps), wp, wdt,
                                         lp, ldt, gp, gdt, B, L_max, dl, Hs, Hn, Hkv, d,
                                         int(window), float(scale), out.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected the decode arguments (rc %d)" % rc)
        return out


    # backward: gradients of sum(d_out * O) with respect to every input
    def gdla_attn_bwd(self, q_sig, q_noise, k, v, lam, gate, d_out, window: int = 0,
                      causal: bool = True, scale=None) -> dict:
        """Gradients of the GDLA forward for upstream gradient d_out [B,T,Hs*d].

        Returns float64 arrays dq_sig [B,T,Hs,d], dq_noise [B,T,Hn,d],
        dk, dv [B,T,Hkv,d], dlam [B,T,Hs], dgate [B,T,Hs*d].
        """
        qs, qsp, qsdt = _arr(q_sig)
        qn, qnp, qndt = _arr(q_noise)
        ka, kp, kdt = _arr(k)
        va, vp, vdt = _arr(v)
        la, lp, ldt = _arr(lam)
        ga, gp, gdt = _arr(gate)
        da, dp, ddt = _arr(d_out)
        B, T, Hs, d = qs.shape
        Hn = qn.shape[2]
        Hkv = ka.shape[2]
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        out = {"dq_sig": np.empty((B, T, Hs, d)), "dq_noise": np.empty((B, T, Hn, d)),
               "dk": np.empty((B, T, Hkv, d)), "dv": np.empty((B, T, Hkv, d)),
               "dlam": np.empty((B, T, Hs)), "dgate": np.empty((B, T, Hs * d))}
        rc = self.lib.gdla_oracle_attn_bwd(qsp, qsdt, qnp, qndt, kp, kdt, vp, vdt, lp, ldt, gp,
                                           gdt, dp, ddt, B, T, Hs, Hn, Hkv, d, int(window),
                                           int(bool(causal)), float(scale),
                                           *(out[n].ctypes.data for n in
                                             ("dq_sig", "dq_noise", "dk", "dv", "dlam", "dgate")))
        if rc != 0:
            raise ValueError("oracle rejected the backward arguments (rc %d)" % rc)
        return out


_default = None


def default() -> Oracle:
    """The oracle built from ``gdla_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def rmsnorm(*a, **k):
    return default().rmsnorm(*a, **k)


def kv_expand(*a, **k):
    return default().kv_expand(*a, **k)


def attention_path(*a, **k):
    return default().attention_path(*a, **k)


def differential_gate(*a, **k):
    return default().differential_gate(*a, **k)


def gdla_attn(*a, **k):
    return default().gdla_attn(*a, **k)


def gdla_attn_rows(*a, **k):
    return default().gdla_attn_rows(*a, **k)


def decode(*a, **k):
    return default().decode(*a, **k)


def gdla_attn_bwd(*a, **k):
    return default().gdla_attn_bwd(*a, **k)
