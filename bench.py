"""Throughput of the GDLA forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input.
The default workload is the latent-KV layer (B=1, T=32768, 64 signal / 16
noise / 16 KV heads, d=128, full causal): RMSNorm + W^KV_b expand of the 512-d
KV latent, then the fused GDLA attention.  Other workloads (--workload window,
full, tiny, long_full, long_window) time the attention alone.

Metric: TFLOP/s of algorithmic work (attention: 4*d FLOPs per kept (query,key)
pair per query head; expand: 2*512*4096 per token), plus tokens/s.  Inputs are
resident in HBM and larger than L2 (no flush needed); timing uses CUDA events
on the launching stream with W untimed warm-up steps.  Multi-GPU runs are
independent replicas (the forward pass has no cross-GPU exchange); the time is
the maximum over ranks and the value is all ranks' work over that time.

--impl reference times the float64 CPU oracle (the only other implementation of
this method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDLA attn fwd TFLOP/s and tokens/s on 1 B200; % of bf16 tensor or HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        self.path = os.path.join("/tmp", "gdla_clocks_%d.csv" % os.getpid())
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", gpu_id], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value across ranks (all ranks call this in the same order)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Each replica draws its own inputs (same recipe, seed = rank)."""
    return int(rank)


def _gpu_id(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # pragma: no cover
        return str(dev.index or 0)


def run_ours(args):
    import torch
    import torch.distributed as dist

    import grouped_differential_attention_gdla_b200 as gdla
    from grouped_differential_attention_gdla_b200.build import build
    from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, make_inputs

    world, rank, local = _dist()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    gdla.load_library()
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    x = make_inputs(wl, seed=replica_seed(rank), device=dev)
    n_tok = wl.B * wl.T
    stream = torch.cuda.current_stream(dev)
    if wl.latent:
        kbuf = torch.empty((n_tok, wl.Hkv, wl.d), dtype=torch.bfloat16, device=dev)
        vbuf = torch.empty_like(kbuf)
    out = torch.empty((wl.B, wl.T, wl.Hs * wl.d), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(ev=None, inp=x, strm=None):
        st = stream if strm is None else strm
        if wl.latent:
            gdla.gdla_kv_expand(inp["c_kv"], inp["w_kvb"], None, eps=wl.eps, d_head=wl.d,
                                k_out=kbuf, v_out=vbuf, d_status=status, stream=st)
            k = kbuf.view(wl.B, wl.T, wl.Hkv, wl.d)
            v = vbuf.view(wl.B, wl.T, wl.Hkv, wl.d)
        else:
            k, v = inp["k"], inp["v"]
        if ev is not None:
            ev[0].record(st)
        gdla.gdla_attn_fwd(inp["q_sig"], inp["q_noise"], k, v, inp["lam"], inp["gate"],
                           window=wl.window, causal=wl.causal, out=out, d_status=status,
                           stream=st)
        if ev is not None:
            ev[1].record(st)

    launches_per_step = 2 if wl.latent else 1
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError("kernel reported status %d during warm-up" % int(status.item()))

    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(_gpu_id(torch, dev)) if rank == 0 else None
    time.sleep(0.25 if sampler else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(args.steps):
        step(attn_ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    ms = t0.elapsed_time(t1)
    attn_ms = sum(a.elapsed_time(b) for a, b in attn_ev) / args.steps
    if int(status.item()) != 0:
        raise RuntimeError("kernel reported status %d" % int(status.item()))
    ms = max_over_ranks(ms, world, dev)

    # ---- end to end through the public API from pinned host memory.  Every
    # step copies its inputs host->device and its output device->host inside
    # the timed region; steps are pipelined over three streams (upload of step
    # i+1 and download of step i-1 overlap the kernels of step i), with two
    # device buffers for inputs and outputs.
    e2e_steps = max(2, min(args.steps, 6))
    host = {n: t.to("cpu").pin_memory() for n, t in x.items()}
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out.numel() * out.element_size()
    dev_in = [{n: torch.empty_like(t) for n, t in x.items()} for _ in range(2)]
    dev_out = [out, torch.empty_like(out)]
    s_up, s_run, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("up", "run", "down")}
    for k in ev:
        for e in ev[k]:
            e.record(stream)

    def e2e_step(i):
        nonlocal out
        bsel = i % 2
        s_up.wait_event(ev["run"][bsel])           # inputs of step i-2 consumed
        with torch.cuda.stream(s_up):
            for n, t in host.items():
                dev_in[bsel][n].copy_(t, non_blocking=True)
            ev["up"][bsel].record(s_up)
        s_run.wait_event(ev["up"][bsel])
        s_run.wait_event(ev["down"][bsel])         # output of step i-2 downloaded
        with torch.cuda.stream(s_run):
            out = dev_out[bsel]
            step(inp=dev_in[bsel], strm=s_run)
            ev["run"][bsel].record(s_run)
        s_down.wait_event(ev["run"][bsel])
        with torch.cuda.stream(s_down):
            out_host[bsel].copy_(dev_out[bsel], non_blocking=True)
            ev["down"][bsel].record(s_down)

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(e2e_steps):
        e2e_step(i)
    s_down.wait_stream(s_run)
    e1.record(s_down)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    if world > 1:
        dist.barrier()
    out = dev_out[0]

    step_flops = wl.attn_flops() + (wl.expand_flops() if wl.latent else 0)
    value = step_flops * args.steps * world / (ms * 1e-3) / 1e12
    e2e_value = step_flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12
    peaks, peak_src = _peaks()
    if wl.window > 0:
        bound, unit_r = "hbm", "GB/s"
        achieved = wl.attn_bytes() / (attn_ms * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
    else:
        bound, unit_r = "tensor", "TFLOP/s"
        achieved = wl.attn_flops() / (attn_ms * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops_sustained"])
    traffic = _traffic_from_profiles(wl.name)
    result = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "tokens_per_s": round(n_tok * args.steps * world / (ms * 1e-3), 1),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 inputs, sigmoid lambda/gate)",
        "config": {
            "workload": wl.name, "B": wl.B, "T": wl.T, "Hs": wl.Hs, "Hn": wl.Hn, "Hkv": wl.Hkv,
            "d": wl.d, "window": wl.window, "causal": wl.causal, "latent_kv": wl.latent,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (%.0f MB per step)" % (
                (wl.attn_bytes() + (wl.expand_bytes() if wl.latent else 0)) / 1e6),
        },
        "roofline": {
            "kernel": "gdla_attn_fwd_kernel",
            "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit_r,
            "frac": round(achieved / peak, 4),
            "peak_source": "%s %s" % (peak_src, "hbm_gbs" if bound == "hbm" else
                                      "bf16_tflops_sustained"),
            "avg_launch_ms": round(attn_ms, 4),
            "traffic": traffic,
        },
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "mode": "pinned host buffers, copies pipelined with compute over 3 streams"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, x, seconds=args.cpu_seconds)
    del host, out_host, dev_in, dev_out
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def _strip_comments(src):
    """C/C++ source without its comments or blank-line differences."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def _csrc_hash():
    """Hash of the CUDA sources' code (comments excluded), to tell whether
    profiled counters still apply to the kernels being timed."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "grouped_differential_attention_gdla_b200",
                                           "csrc", "*"))):
        with open(f, encoding="utf-8") as fh:
            h.update(_strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def _traffic_from_profiles(name):
    """DRAM bytes (read + write) per attention launch from a committed ncu
    summary under profiles/ (a line "traffic: workload=<w> csrc=<hash>
    bytes=<n>"), or None when none matches this workload and these sources."""
    import glob
    import re
    want = _csrc_hash()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as f:
            for m in re.finditer(r"traffic: workload=(\S+) csrc=(\S+) bytes=(\d+)", f.read()):
                if m.group(1) == name and m.group(2) == want:
                    return int(m.group(3))
    return None


def _oracle_sample(wl, x, seconds):
    """Time the float64 oracle on a bounded sample of the workload.

    Sample: query rows drawn uniformly from the first `span` tokens of batch 0
    (all heads), plus, for the latent workload, the RMSNorm + expand of the
    tokens those rows need.  Returns (flops, elapsed_s, description).
    """
    import numpy as np
    import torch

    import oracle

    rng = np.random.default_rng(0)
    span = min(wl.T, 4096)
    # rows per pass: a sliding-window row costs W pairs, a causal row up to span
    n_rows = 256 if wl.window > 0 else 8
    total_flops, total_s, rows_done = 0, 0.0, 0
    cpu = {}
    for n in ("c_kv", "w_kvb", "k", "v"):
        if n in x:
            t = x[n]
            cpu[n] = (t[:span] if n == "c_kv" else (t[:1, :span] if n in ("k", "v") else t)).cpu()
    kv_cache = None
    while total_s < seconds:
        t0 = time.perf_counter()
        flops = 0
        if wl.latent:
            chat = oracle.rmsnorm(cpu["c_kv"], None, wl.eps)
            rk, rv = oracle.kv_expand(chat, cpu["w_kvb"], wl.Hkv, wl.d, wl.d)
            k = rk.reshape(1, span, wl.Hkv, wl.d)
            v = rv.reshape(1, span, wl.Hkv, wl.d)
            flops += 2 * span * wl.d_latent * wl.Hkv * 2 * wl.d
        else:
            k, v = cpu["k"], cpu["v"]
        rows = np.sort(rng.integers(0, span, n_rows))
        idx = torch.as_tensor(rows, device=x["q_sig"].device)
        g = lambda t: t[0].index_select(0, idx).cpu()
        oracle.gdla_attn_rows(g(x["q_sig"]), g(x["q_noise"]), k, v, g(x["lam"]), g(x["gate"]),
                              rows, window=wl.window, causal=wl.causal)
        for i in rows:
            kept = min(int(i) + 1, wl.window) if wl.window > 0 else int(i) + 1
            flops += 4 * wl.d * (wl.Hs + wl.Hn) * kept
        total_s += time.perf_counter() - t0
        total_flops += flops
        rows_done += n_rows
    desc = ("%d query rows (all %d heads) drawn uniformly from the first %d tokens%s, float64 "
            "oracle" % (rows_done, wl.Hs + wl.Hn, span,
                        ", plus RMSNorm+W^KV_b expand of those %d tokens per pass" % span
                        if wl.latent else ""))
    return total_flops, total_s, desc


def cpu_baseline(wl, x, seconds=15.0):
    flops, s, desc = _oracle_sample(wl, x, seconds)
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(flops / s / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle", "sample": desc, "seconds": round(s, 2)}


def run_reference(args):
    """Reference arm: the float64 CPU oracle on a bounded sample per step."""
    world, rank, local = _dist()
    if rank != 0:
        return
    import torch

    from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, make_inputs
    import oracle

    oracle.build()
    wl = WORKLOADS[args.workload]
    # inputs drawn on the CPU in the same recipe; only the sampled slices are used
    x = make_inputs(wl, seed=0, device="cpu", T=min(wl.T, 4096), B=1)
    per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        _oracle_sample(wl, x, per_step / 4)
    flops, secs = 0, 0.0
    desc = ""
    for _ in range(args.steps):
        f, s, desc = _oracle_sample(wl, x, per_step)
        flops += f
        secs += s
    value = flops / secs / 1e12
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    n_tok = wl.B * wl.T
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3 / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same recipe, CPU draw)",
        "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "Hs": wl.Hs, "Hn": wl.Hn,
                   "Hkv": wl.Hkv, "d": wl.d, "window": wl.window, "causal": wl.causal,
                   "latent_kv": wl.latent},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": desc + " (per step)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
        "note": "float64 CPU oracle on %d host threads; tokens/s of the full workload would be "
                "%.3g" % (threads, n_tok * value * 1e12 / max(1, wl.attn_flops())),
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="latent",
                    choices=["latent", "window", "full", "tiny", "long_full", "long_window"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
