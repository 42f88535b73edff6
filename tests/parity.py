"""Shared helpers for the GPU parity tests: the per-tensor tolerance and row
sampling.  The tolerance is the one the forward pass is held to everywhere:
max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3 over each checked tensor.

With GDLA_PARITY_LOG=<path> set, every checked tensor's error statistics are
appended to <path> as one JSON line (tests/parity_report.py turns the file
into a table)."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

RTOL = 1e-2
ATOL = 1e-3


def error_stats(gpu, ref) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(gpu - ref)
    idx = int(np.argmax(diff)) if diff.size else 0
    return {
        "max_abs_err": float(diff.max()) if diff.size else 0.0,
        "max_abs_ref": float(np.abs(ref).max()) if ref.size else 0.0,
        "mean_abs_err": float(diff.mean()) if diff.size else 0.0,
        "rms_err": float(np.sqrt((diff ** 2).mean())) if diff.size else 0.0,
        "argmax": np.unravel_index(idx, diff.shape) if diff.size else (),
        "finite": bool(np.isfinite(gpu).all()),
    }


def _log(what: str, st: dict, tol: float, n_rows: int) -> None:
    path = os.environ.get("GDLA_PARITY_LOG")
    if not path:
        return
    rec = {"what": what, "elements": n_rows, "tol": tol,
           **{k: (list(map(int, v)) if k == "argmax" else v) for k, v in st.items()}}
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def assert_parity(gpu, ref, what: str) -> dict:
    st = error_stats(gpu, ref)
    tol = RTOL * st["max_abs_ref"] + ATOL
    _log(what, st, tol, int(np.asarray(ref).size))
    assert st["finite"], f"{what}: non-finite GPU output"
    assert st["max_abs_err"] <= tol, (
        f"{what}: max|gpu-oracle| = {st['max_abs_err']:.4e} > tol {tol:.4e} "
        f"(max|oracle| {st['max_abs_ref']:.3e}, mean err {st['mean_abs_err']:.2e}, "
        f"at {st['argmax']})")
    return st


def sample_rows(B: int, T: int, n_random: int, seed: int = 0, extra=()) -> np.ndarray:
    """Flat row indices b*T+i: block edges, the first and last rows of every
    batch element, and random rows."""
    rng = np.random.default_rng(seed)
    pick = set()
    for b in range(B):
        for i in (0, 1, 2, 63, 64, 127, 128, 129, 255, 256, T // 2, T - 129, T - 128, T - 2,
                  T - 1, *extra):
            if 0 <= i < T:
                pick.add(b * T + i)
    if n_random:
        pick.update(rng.integers(0, B * T, size=n_random).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def gather_rows(t: torch.Tensor, rows) -> torch.Tensor:
    """Rows of a [B, T, ...] tensor by flat index, copied to the host."""
    B, T = t.shape[0], t.shape[1]
    flat = t.reshape(B * T, *t.shape[2:])
    idx = torch.as_tensor(rows, device=t.device, dtype=torch.long)
    return flat.index_select(0, idx).cpu()
