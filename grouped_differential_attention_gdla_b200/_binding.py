"""ctypes binding of libgdla.so: argument marshalling only.

Every step of the forward pass runs in the library's CUDA kernels; this module
checks tensor dtypes, shapes, devices and contiguity, passes raw device
pointers, sizes and the current CUDA stream, and turns status codes into
exceptions.  There is no fallback: without the compiled library every call
raises.

Device-side failures (a pipeline wait that gave up) land in an int32 status
word.  Calls that pass no ``d_status`` share one word per device; read it with
``check_status()`` after the stream has passed the calls, or set
``GDLA_SYNC_CHECK=1`` to synchronise and check after every call.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdla.so")

GDLA_OK = 0
GDLA_ERR_INVALID_ARG = -1
GDLA_ERR_UNSUPPORTED = -2
GDLA_ERR_ALIGNMENT = -3
GDLA_ERR_CUDA = -4
GDLA_ERR_TIMEOUT = -5

# every symbol include/gdla.h declares
EXPORTED = ("gdla_version", "gdla_status_string", "gdla_kv_expand", "gdla_attn_fwd",
            "gdla_attn_fwd_sp", "gdla_latent_rmsnorm", "gdla_decode_workspace_bytes",
            "gdla_decode_fwd", "gdla_selftest_wait_timeout", "gdla_decode_fwd_noalloc",
            "gdla_attn_fwd_rope", "gdla_attn_bwd_workspace_bytes", "gdla_attn_bwd")

_lib = None
# One status word per device, used when a caller passes none (see check_status).
_default_status = {}


class GDLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {gdla_status_string(code)} (status {code})")


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libgdla.so (raises when it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"libgdla.so not found at {p}; build it with "
            "`python -m grouped_differential_attention_gdla_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.gdla_version.argtypes = []
    lib.gdla_version.restype = i32
    lib.gdla_status_string.argtypes = [i32]
    lib.gdla_status_string.restype = ctypes.c_char_p
    lib.gdla_kv_expand.argtypes = [vp, vp, vp, f32, vp, vp, i64, i32, i32, i32, vp, vp]
    lib.gdla_kv_expand.restype = i32
    lib.gdla_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i64,
                                  i32, f32, vp, vp]
    lib.gdla_attn_fwd.restype = i32
    lib.gdla_attn_fwd_sp.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i64, i32, i32, i32,
                                     i32, i64, f32, vp, vp]
    lib.gdla_attn_fwd_sp.restype = i32
    lib.gdla_attn_fwd_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                       i32, i32, i32, i64, i32, f32, vp, vp]
    lib.gdla_attn_fwd_rope.restype = i32
    lib.gdla_attn_bwd_workspace_bytes.argtypes = [i32, i64, i32, i32, i32]
    lib.gdla_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.gdla_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64,
                                  i32, i32, i32, i32, i64, i32, f32, vp, ctypes.c_size_t, vp, vp]
    lib.gdla_attn_bwd.restype = i32
    lib.gdla_latent_rmsnorm.argtypes = [vp, vp, f32, vp, i64, i32, vp, vp]
    lib.gdla_latent_rmsnorm.restype = i32
    lib.gdla_decode_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i64]
    lib.gdla_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.gdla_decode_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                    i32, i64, f32, vp, ctypes.c_size_t, vp, vp]
    lib.gdla_decode_fwd.restype = i32
    lib.gdla_selftest_wait_timeout.argtypes = [vp, i64, vp]
    lib.gdla_decode_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                            i32, i32, i32, i64, f32, vp, vp]
    lib.gdla_decode_fwd_noalloc.restype = i32
    lib.gdla_selftest_wait_timeout.restype = i32
    if path is None:
        _lib = lib
    return lib


def gdla_version() -> int:
    return load_library().gdla_version()


def gdla_status_string(code: int) -> str:
    return load_library().gdla_status_string(int(code)).decode()


def _check(t: torch.Tensor, name: str, shape=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _same_device(device: torch.device, tensors) -> None:
    for name, t in tensors:
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device} like the other inputs")


def _status_ptr(d_status: Optional[torch.Tensor], device: torch.device) -> int:
    """Device pointer of the int32 status word; the per-device default word
    when the caller passes none."""
    if d_status is None:
        d_status = _default_status.get(device)
        if d_status is None:
            d_status = torch.zeros(1, dtype=torch.int32, device=device)
            _default_status[device] = d_status
    if not isinstance(d_status, torch.Tensor) or d_status.dtype != torch.int32:
        raise ValueError("d_status must be an int32 tensor")
    if d_status.device != device:
        raise ValueError(f"d_status is on {d_status.device}, expected {device}")
    if d_status.numel() < 1:
        raise ValueError("d_status must hold at least one element")
    return d_status.data_ptr()


def check_status(device=None, d_status: Optional[torch.Tensor] = None) -> None:
    """Synchronise `device` and raise GDLAError if a kernel reported a failure
    in `d_status` (default: the word used by calls that passed none).  The
    word is cleared afterwards, so a later check reports only later calls."""
    if d_status is None:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        d_status = _default_status.get(dev)
        if d_status is None:
            return
    torch.cuda.synchronize(d_status.device)
    code = int(d_status[0].item())
    if code != GDLA_OK:
        d_status.zero_()
        raise GDLAError(code, "device-side status")


def _sync_check_enabled() -> bool:
    return os.environ.get("GDLA_SYNC_CHECK", "0") not in ("", "0")


def _stream_ptr(device: torch.device, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def gdla_kv_expand(c_kv: torch.Tensor, w_kvb: torch.Tensor, rms_w: Optional[torch.Tensor] = None,
                   eps: float = 1e-6, d_head: int = 128, k_out: Optional[torch.Tensor] = None,
                   v_out: Optional[torch.Tensor] = None, d_status: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """RMSNorm(c_kv) @ W^KV_b split into K, V [N, Hkv, d_head] (bf16, CUDA)."""
    if c_kv.dim() != 2 or w_kvb.dim() != 2:
        raise ValueError("c_kv must be [N, d_latent] and w_kvb [d_latent, Hkv*2*d_head]")
    n, dl = c_kv.shape
    if w_kvb.shape[0] != dl or w_kvb.shape[1] % (2 * d_head) != 0:
        raise ValueError("w_kvb must be [d_latent, Hkv*2*d_head]")
    hkv = w_kvb.shape[1] // (2 * d_head)
    if k_out is None:
        k_out = torch.empty((n, hkv, d_head), dtype=torch.bfloat16, device=c_kv.device)
    if v_out is None:
        v_out = torch.empty((n, hkv, d_head), dtype=torch.bfloat16, device=c_kv.device)
    pc = _check(c_kv, "c_kv")
    pw = _check(w_kvb, "w_kvb")
    pr = _check(rms_w, "rms_w", (dl,)) if rms_w is not None else None
    pk = _check(k_out, "k_out", (n, hkv, d_head))
    pv = _check(v_out, "v_out", (n, hkv, d_head))
    _same_device(c_kv.device, [("w_kvb", w_kvb), ("rms_w", rms_w), ("k_out", k_out),
                               ("v_out", v_out)])
    ps = _status_ptr(d_status, c_kv.device)
    rc = load_library().gdla_kv_expand(pc, pr, pw, float(eps), pk, pv, n, dl, hkv, d_head, ps,
                                       _stream_ptr(c_kv.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_kv_expand")
    if _sync_check_enabled():
        check_status(c_kv.device, d_status)
    return k_out, v_out


def gdla_attn_fwd(q_sig: torch.Tensor, q_noise: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                  lam: torch.Tensor, gate: torch.Tensor, window: int = 0, causal: bool = True,
                  scale: float = 0.0, out: Optional[torch.Tensor] = None,
                  d_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Fused GDLA attention forward; returns out [B, T, Hs*d] (bf16, CUDA).

    q_sig [B,T,Hs,d], q_noise [B,T,Hn,d], k/v [B,T,Hkv,d], lam [B,T,Hs],
    gate [B,T,Hs*d].  window 0 = full causal; scale <= 0 means 1/sqrt(d).
    """
    if q_sig.dim() != 4:
        raise ValueError("q_sig must be [B, T, Hs, d]")
    B, T, Hs, d = q_sig.shape
    Hn = q_noise.shape[2] if q_noise.dim() == 4 else -1
    Hkv = k.shape[2] if k.dim() == 4 else -1
    if out is None:
        out = torch.empty((B, T, Hs * d), dtype=torch.bfloat16, device=q_sig.device)
    ptrs = [
        _check(q_sig, "q_sig"),
        _check(q_noise, "q_noise", (B, T, Hn, d)),
        _check(k, "k", (B, T, Hkv, d)),
        _check(v, "v", (B, T, Hkv, d)),
        _check(lam, "lam", (B, T, Hs)),
        _check(gate, "gate", (B, T, Hs * d)),
        _check(out, "out", (B, T, Hs * d)),
    ]
    _same_device(q_sig.device, [("q_noise", q_noise), ("k", k), ("v", v), ("lam", lam),
                                 ("gate", gate), ("out", out)])
    ps = _status_ptr(d_status, q_sig.device)
    rc = load_library().gdla_attn_fwd(*ptrs, B, T, Hs, Hn, Hkv, d, int(window), int(bool(causal)),
                                      float(scale), ps, _stream_ptr(q_sig.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_attn_fwd")
    if _sync_check_enabled():
        check_status(q_sig.device, d_status)
    return out


def gdla_attn_fwd_rope(q_sig: torch.Tensor, q_noise: torch.Tensor, q_rope_sig: torch.Tensor,
                       q_rope_noise: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       k_rope: torch.Tensor, lam: torch.Tensor, gate: torch.Tensor,
                       window: int = 0, causal: bool = True, scale: float = 0.0,
                       out: Optional[torch.Tensor] = None,
                       d_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """GDLA attention forward with the decoupled rotary term; returns out
    [B, T, Hs*d].

    As gdla_attn_fwd, plus q_rope_sig [B,T,Hs,dr], q_rope_noise [B,T,Hn,dr]
    and k_rope [B,T,dr] (one rotary key per token shared by every head;
    dr = 64).  scale <= 0 means 1/sqrt(d + dr).
    """
    if q_sig.dim() != 4 or k_rope.dim() != 3:
        raise ValueError("q_sig must be [B, T, Hs, d] and k_rope [B, T, d_rope]")
    B, T, Hs, d = q_sig.shape
    Hn = q_noise.shape[2] if q_noise.dim() == 4 else -1
    Hkv = k.shape[2] if k.dim() == 4 else -1
    dr = k_rope.shape[2]
    if out is None:
        out = torch.empty((B, T, Hs * d), dtype=torch.bfloat16, device=q_sig.device)
    ptrs = [
        _check(q_sig, "q_sig"),
        _check(q_noise, "q_noise", (B, T, Hn, d)),
        _check(q_rope_sig, "q_rope_sig", (B, T, Hs, dr)),
        _check(q_rope_noise, "q_rope_noise", (B, T, Hn, dr)),
        _check(k, "k", (B, T, Hkv, d)),
        _check(v, "v", (B, T, Hkv, d)),
        _check(k_rope, "k_rope", (B, T, dr)),
        _check(lam, "lam", (B, T, Hs)),
        _check(gate, "gate", (B, T, Hs * d)),
        _check(out, "out", (B, T, Hs * d)),
    ]
    _same_device(q_sig.device, [("q_noise", q_noise), ("q_rope_sig", q_rope_sig),
                                 ("q_rope_noise", q_rope_noise), ("k", k), ("v", v),
                                 ("k_rope", k_rope), ("lam", lam), ("gate", gate), ("out", out)])
    ps = _status_ptr(d_status, q_sig.device)
    rc = load_library().gdla_attn_fwd_rope(*ptrs, B, T, Hs, Hn, Hkv, d, dr, int(window),
                                           int(bool(causal)), float(scale), ps,
                                           _stream_ptr(q_sig.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_attn_fwd_rope")
    if _sync_check_enabled():
        check_status(q_sig.device, d_status)
    return out


def gdla_attn_bwd_workspace_bytes(B: int, T: int, Hs: int, Hn: int, d: int) -> int:
    """Device scratch bytes gdla_attn_bwd needs for these shapes."""
    return int(load_library().gdla_attn_bwd_workspace_bytes(B, T, Hs, Hn, d))


def gdla_attn_bwd(q_sig: torch.Tensor, q_noise: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                  lam: torch.Tensor, gate: torch.Tensor, d_out: torch.Tensor, window: int = 0,
                  causal: bool = True, scale: float = 0.0, grads: Optional[dict] = None,
                  workspace: Optional[torch.Tensor] = None,
                  d_status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Gradients of gdla_attn_fwd for the upstream gradient d_out [B,T,Hs*d].

    Returns a dict of bf16 CUDA tensors dq_sig, dq_noise, dk, dv, dlam, dgate
    (written into `grads` when given).  The scratch comes from `workspace` (a
    uint8 CUDA tensor) or, when None, is allocated here with torch.
    """
    if q_sig.dim() != 4:
        raise ValueError("q_sig must be [B, T, Hs, d]")
    B, T, Hs, d = q_sig.shape
    Hn = q_noise.shape[2] if q_noise.dim() == 4 else -1
    Hkv = k.shape[2] if k.dim() == 4 else -1
    dev = q_sig.device
    shapes = {"dq_sig": (B, T, Hs, d), "dq_noise": (B, T, Hn, d), "dk": (B, T, Hkv, d),
              "dv": (B, T, Hkv, d), "dlam": (B, T, Hs), "dgate": (B, T, Hs * d)}
    if grads is None:
        grads = {n: torch.empty(sh, dtype=torch.bfloat16, device=dev) for n, sh in shapes.items()}
    need = gdla_attn_bwd_workspace_bytes(B, T, Hs, Hn, d) if B > 0 and T > 0 else 0
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if workspace.dtype != torch.uint8 or workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor on the inputs' device")
    ptrs = [
        _check(q_sig, "q_sig"),
        _check(q_noise, "q_noise", (B, T, Hn, d)),
        _check(k, "k", (B, T, Hkv, d)),
        _check(v, "v", (B, T, Hkv, d)),
        _check(lam, "lam", (B, T, Hs)),
        _check(gate, "gate", (B, T, Hs * d)),
        _check(d_out, "d_out", (B, T, Hs * d)),
    ] + [_check(grads[n], n, shapes[n]) for n in shapes]
    _same_device(dev, [("q_noise", q_noise), ("k", k), ("v", v), ("lam", lam), ("gate", gate),
                       ("d_out", d_out)] + [(n, grads[n]) for n in shapes])
    ps = _status_ptr(d_status, dev)
    rc = load_library().gdla_attn_bwd(*ptrs, B, T, Hs, Hn, Hkv, d, int(window), int(bool(causal)),
                                      float(scale), workspace.data_ptr(), workspace.numel(), ps,
                                      _stream_ptr(dev, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_attn_bwd")
    if _sync_check_enabled():
        check_status(dev, d_status)
    return grads


def gdla_attn_fwd_sp(q_sig: torch.Tensor, q_noise: torch.Tensor, k: torch.Tensor,
                     v: torch.Tensor, lam: torch.Tensor, gate: torch.Tensor, window: int,
                     kv_prefix: int, scale: float = 0.0, out: Optional[torch.Tensor] = None,
                     d_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Sliding-window GDLA forward on one shard of a sequence split across GPUs.

    q_sig [B,T,Hs,d], q_noise [B,T,Hn,d], lam [B,T,Hs], gate [B,T,Hs*d] hold
    the shard's T tokens; k/v [B, kv_prefix+T, Hkv, d] hold kv_prefix halo
    rows (the previous shard's last keys; 0 on the first shard) and then the
    shard's own.  window in 1..128.  Returns out [B, T, Hs*d].
    """
    if q_sig.dim() != 4:
        raise ValueError("q_sig must be [B, T, Hs, d]")
    B, T, Hs, d = q_sig.shape
    Hn = q_noise.shape[2] if q_noise.dim() == 4 else -1
    Hkv = k.shape[2] if k.dim() == 4 else -1
    if out is None:
        out = torch.empty((B, T, Hs * d), dtype=torch.bfloat16, device=q_sig.device)
    ptrs = [
        _check(q_sig, "q_sig"),
        _check(q_noise, "q_noise", (B, T, Hn, d)),
        _check(k, "k", (B, kv_prefix + T, Hkv, d)),
        _check(v, "v", (B, kv_prefix + T, Hkv, d)),
        _check(lam, "lam", (B, T, Hs)),
        _check(gate, "gate", (B, T, Hs * d)),
        _check(out, "out", (B, T, Hs * d)),
    ]
    _same_device(q_sig.device, [("q_noise", q_noise), ("k", k), ("v", v), ("lam", lam),
                                 ("gate", gate), ("out", out)])
    ps = _status_ptr(d_status, q_sig.device)
    rc = load_library().gdla_attn_fwd_sp(*ptrs, B, T, int(kv_prefix), Hs, Hn, Hkv, d, int(window),
                                         float(scale), ps, _stream_ptr(q_sig.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_attn_fwd_sp")
    if _sync_check_enabled():
        check_status(q_sig.device, d_status)
    return out


def gdla_latent_rmsnorm(c_kv: torch.Tensor, rms_w: Optional[torch.Tensor] = None,
                        eps: float = 1e-6, out: Optional[torch.Tensor] = None,
                        d_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """RMSNorm of KV latents entering the decode cache: c_kv [..., d_latent]
    (bf16, CUDA) -> out of the same shape (may be a view into the cache)."""
    dl = c_kv.shape[-1]
    n = c_kv.numel() // dl if dl else 0
    if out is None:
        out = torch.empty_like(c_kv)
    pc = _check(c_kv, "c_kv")
    po = _check(out, "out", tuple(c_kv.shape))
    pr = _check(rms_w, "rms_w", (dl,)) if rms_w is not None else None
    _same_device(c_kv.device, [("rms_w", rms_w), ("out", out)])
    ps = _status_ptr(d_status, c_kv.device)
    rc = load_library().gdla_latent_rmsnorm(pc, pr, float(eps), po, n, dl, ps,
                                            _stream_ptr(c_kv.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_latent_rmsnorm")
    return out


def gdla_decode_workspace_bytes(B: int, L_max: int, Hs: int, Hn: int, d_latent: int = 512,
                                window: int = 0) -> int:
    """Device scratch bytes gdla_decode_fwd needs for these shapes."""
    return int(load_library().gdla_decode_workspace_bytes(B, L_max, Hs, Hn, d_latent,
                                                         int(window)))


def gdla_decode_fwd(q_sig: torch.Tensor, q_noise: torch.Tensor, c_hat: torch.Tensor,
                    cache_len: torch.Tensor, w_kvb: torch.Tensor, lam: torch.Tensor,
                    gate: torch.Tensor, window: int = 0, scale: float = 0.0,
                    out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    d_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """GDLA forward of the newest token of each sequence over its latent cache.

    q_sig [B,Hs,d], q_noise [B,Hn,d], c_hat [B,L_max,d_latent] (RMSNorm'd
    latents, gdla_latent_rmsnorm), cache_len int32 [B] on the device,
    w_kvb [d_latent, Hn*2d], lam [B,Hs], gate [B,Hs*d].  Returns out [B, Hs*d].
    The scratch comes from `workspace` (a uint8 CUDA tensor) or, when None,
    is allocated here with torch (the library itself never allocates).
    """
    if q_sig.dim() != 3 or c_hat.dim() != 3:
        raise ValueError("q_sig must be [B, Hs, d] and c_hat [B, L_max, d_latent]")
    B, Hs, d = q_sig.shape
    Hn = q_noise.shape[1] if q_noise.dim() == 3 else -1
    L_max, dl = c_hat.shape[1], c_hat.shape[2]
    hkv = w_kvb.shape[1] // (2 * d) if w_kvb.dim() == 2 else -1
    if out is None:
        out = torch.empty((B, Hs * d), dtype=torch.bfloat16, device=q_sig.device)
    need = gdla_decode_workspace_bytes(B, L_max, Hs, Hn, dl, window) if B > 0 else 0
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q_sig.device)
    if workspace.dtype != torch.uint8 or workspace.device != q_sig.device or \
            not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor on the inputs' device")
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or \
            not cache_len.is_contiguous():
        raise ValueError("cache_len must be a contiguous int32 tensor of shape [B]")
    ptrs = [
        _check(q_sig, "q_sig"),
        _check(q_noise, "q_noise", (B, Hn, d)),
        _check(c_hat, "c_hat"),
    ]
    pw = _check(w_kvb, "w_kvb", (dl, hkv * 2 * d))
    pl = _check(lam, "lam", (B, Hs))
    pg = _check(gate, "gate", (B, Hs * d))
    po = _check(out, "out", (B, Hs * d))
    _same_device(q_sig.device, [("q_noise", q_noise), ("c_hat", c_hat), ("cache_len", cache_len),
                                 ("w_kvb", w_kvb), ("lam", lam), ("gate", gate), ("out", out)])
    ps = _status_ptr(d_status, q_sig.device)
    rc = load_library().gdla_decode_fwd(*ptrs, cache_len.data_ptr(), pw, pl, pg, po, B, L_max, Hs,
                                        Hn, hkv, d, dl, int(window), float(scale),
                                        workspace.data_ptr(), workspace.numel(), ps,
                                        _stream_ptr(q_sig.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_decode_fwd")
    if _sync_check_enabled():
        check_status(q_sig.device, d_status)
    return out


# Size of the scratch array compiled into libgdla.so for gdla_decode_fwd_noalloc.
DECODE_NOALLOC_SCRATCH_BYTES = 16 << 20


def gdla_decode_fwd_noalloc(q_sig: torch.Tensor, q_noise: torch.Tensor, c_hat: torch.Tensor,
                            cache_len: torch.Tensor, w_kvb: torch.Tensor, lam: torch.Tensor,
                            gate: torch.Tensor, out: torch.Tensor, window: int = 0,
                            scale: float = 0.0, d_status: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """gdla_decode_fwd without a workspace, for callers that cannot allocate.

    The decode's scratch comes from an array compiled into the library
    (DECODE_NOALLOC_SCRATCH_BYTES per GPU), so neither the library nor this
    wrapper allocates device memory: the caller passes every input and `out`
    [B, Hs*d].  A d_status of None passes no status word.  Shapes needing more
    scratch than the array holds raise GDLAError (GDLA_ERR_UNSUPPORTED).  All
    calls on a device share the array: calls that overlap on the GPU race.
    """
    if q_sig.dim() != 3 or c_hat.dim() != 3:
        raise ValueError("q_sig must be [B, Hs, d] and c_hat [B, L_max, d_latent]")
    B, Hs, d = q_sig.shape
    Hn = q_noise.shape[1] if q_noise.dim() == 3 else -1
    L_max, dl = c_hat.shape[1], c_hat.shape[2]
    hkv = w_kvb.shape[1] // (2 * d) if w_kvb.dim() == 2 else -1
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or \
            not cache_len.is_contiguous():
        raise ValueError("cache_len must be a contiguous int32 tensor of shape [B]")
    ptrs = [
        _check(q_sig, "q_sig"),
        _check(q_noise, "q_noise", (B, Hn, d)),
        _check(c_hat, "c_hat"),
    ]
    pw = _check(w_kvb, "w_kvb", (dl, hkv * 2 * d))
    pl = _check(lam, "lam", (B, Hs))
    pg = _check(gate, "gate", (B, Hs * d))
    po = _check(out, "out", (B, Hs * d))
    _same_device(q_sig.device, [("q_noise", q_noise), ("c_hat", c_hat), ("cache_len", cache_len),
                                 ("w_kvb", w_kvb), ("lam", lam), ("gate", gate), ("out", out)])
    ps = 0
    if d_status is not None:
        _same_device(q_sig.device, [("d_status", d_status)])
        if d_status.dtype != torch.int32:
            raise ValueError("d_status must be an int32 tensor")
        ps = d_status.data_ptr()
    rc = load_library().gdla_decode_fwd_noalloc(*ptrs, cache_len.data_ptr(), pw, pl, pg, po, B,
                                                L_max, Hs, Hn, hkv, d, dl, int(window),
                                                float(scale), ps,
                                                _stream_ptr(q_sig.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_decode_fwd_noalloc")
    return out


def gdla_selftest_wait_timeout(d_status: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self test; d_status (int32 CUDA tensor) gets -5."""
    if d_status.device.type != "cuda" or d_status.dtype != torch.int32:
        raise ValueError("d_status must be an int32 CUDA tensor")
    rc = load_library().gdla_selftest_wait_timeout(d_status.data_ptr(), int(limit_ns),
                                                   _stream_ptr(d_status.device, stream))
    if rc != GDLA_OK:
        raise GDLAError(rc, "gdla_selftest_wait_timeout")
