"""B200-native (sm_100a) forward pass of Grouped Differential Latent Attention.

The compute lives in libgdla.so (hand-written tcgen05/TMA CUDA kernels behind a
C ABI, include/gdla.h); this package is its Python binding.  PyTorch supplies
device memory and streams only.

    gdla_kv_expand(c_kv, w_kvb, rms_w=None, eps=1e-6) -> (K, V)
    gdla_attn_fwd(q_sig, q_noise, k, v, lam, gate, window=0, causal=True) -> out
    gdla_attn_fwd_rope(q_sig, q_noise, q_rope_sig, q_rope_noise, k, v, k_rope, lam, gate)
                            the same with the decoupled rotary term in the score
    gdla_attn_bwd(q_sig, q_noise, k, v, lam, gate, d_out) -> dict of gradients
    gdla_attn_fwd_sp(...)   the sliding window on one shard of a sequence (halo.py
                            exchanges the shards' halo rows between ranks)
    gdla_latent_rmsnorm(c_kv) -> c_hat          cache write: RMSNorm'd KV latents
    gdla_decode_fwd(q_sig, q_noise, c_hat, cache_len, w_kvb, lam, gate) -> out
                            the newest token of each sequence over its latent cache
    gdla_decode_fwd_noalloc(..., out)   the same, with the library's own scratch
                            array, for callers that cannot allocate device memory
"""
from ._binding import (GDLAError, EXPORTED, LIB_PATH, check_status, gdla_attn_bwd,
                       gdla_attn_bwd_workspace_bytes, gdla_attn_fwd,
                       gdla_attn_fwd_rope,
                       gdla_attn_fwd_sp, gdla_decode_fwd, gdla_decode_fwd_noalloc,
                       gdla_decode_workspace_bytes,
                       gdla_kv_expand, gdla_latent_rmsnorm, gdla_selftest_wait_timeout,
                       gdla_status_string, gdla_version, load_library)

__all__ = ["GDLAError", "EXPORTED", "LIB_PATH", "check_status", "gdla_attn_bwd",
           "gdla_attn_bwd_workspace_bytes", "gdla_attn_fwd",
           "gdla_attn_fwd_rope",
           "gdla_attn_fwd_sp", "gdla_decode_fwd", "gdla_decode_fwd_noalloc",
           "gdla_decode_workspace_bytes",
           "gdla_kv_expand", "gdla_latent_rmsnorm", "gdla_selftest_wait_timeout",
           "gdla_status_string", "gdla_version", "load_library"]
