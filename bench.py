"""Throughput of the GDLA forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input.
The default step is the long-context pair of layers (64 signal / 16 noise /
16 KV heads, d=128, B=1): one full-causal layer at T=131072 followed by one
128-token sliding-window layer at T=262144, the 1 full : 3 sliding schedule's
two kinds of attention layer.  --workload latent times the latent-KV layer
(RMSNorm + W^KV_b expand of the 512-d KV latent, then full-causal attention,
T=32768); window, full, tiny, long_full and long_window time one attention
layer alone.

Metric: TFLOP/s of algorithmic work (attention: 4*d FLOPs per kept
(query, key) pair per query head; expand: 2*512*4096 per token), plus
tokens/s.  Inputs are resident in HBM; a step that reads less than twice the
L2 (the 128-token window decode) is preceded by an L2 flush outside its
events.  Timing uses CUDA events on the launching stream with W untimed
warm-up steps, and every library call is bracketed by its own events for the
per-kernel roofline entries.  Decode steps replay one CUDA graph per library
call (--eager launches them directly).  Multi-GPU runs are independent replicas (the forward pass
has no cross-GPU exchange); the time is the maximum over ranks and the value
is all ranks' work over that time.

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

# The layers one step runs, in order.
STEPS = {
    "long": ("long_full", "long_window"),
    "latent": ("latent",),
    "window": ("window",),
    "full": ("full",),
    "tiny": ("tiny",),
    "long_full": ("long_full",),
    "long_window": ("long_window",),
    "decode": ("decode",),
    "decode_window": ("decode_window",),
    "full_rope": ("full_rope",),
    "window_rope": ("window_rope",),
    "bwd_full": ("bwd_full",),
    "bwd_window": ("bwd_window",),
}
# The gradients of a backward layer, in the order they sit in its output buffer.
BWD_GRADS = ("dq_sig", "dq_noise", "dk", "dv", "dlam", "dgate")
# A timed region at least this long runs tensor-bound kernels under the power
# cap, so their fraction is taken against the sustained bf16 peak.
SUSTAINED_AFTER_S = 2.0
# Query rows the CPU sample draws from (the first tokens of batch element 0).
SAMPLE_SPAN = 4096
# Tokens of the causal prefix the oracle's backward runs on for the CPU sample;
# its rows' dQ, dlambda and dG equal the full problem's (they depend on
# earlier keys only).
BWD_SPAN = 512


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


def bwd_grad_shapes(wl):
    return {"dq_sig": (wl.B, wl.T, wl.Hs, wl.d), "dq_noise": (wl.B, wl.T, wl.Hn, wl.d),
            "dk": (wl.B, wl.T, wl.Hkv, wl.d), "dv": (wl.B, wl.T, wl.Hkv, wl.d),
            "dlam": (wl.B, wl.T, wl.Hs), "dgate": (wl.B, wl.T, wl.Hs * wl.d)}


def bwd_grad_views(wl, flat):
    """The six gradients as views of one flat bf16 buffer."""
    out, o = {}, 0
    for n, sh in bwd_grad_shapes(wl).items():
        k = 1
        for e in sh:
            k *= e
        out[n] = flat[o:o + k].view(sh)
        o += k
    return out


def attn_kernel_name(wl) -> str:
    """The kernel gdla_attn_fwd dispatches this layer to (window >= T is full
    causal; windows of 1..128 keys take the union-row kernel)."""
    if wl.bwd:
        return "gdla_attn_bwd"
    if wl.d_rope:
        return "gdla_attn_rope_kernel"
    if wl.causal and 0 < wl.window < wl.T:
        return "gdla_attn_win_kernel" if wl.window <= 128 else "gdla_attn_fwd_kernel<window>"
    return "gdla_attn_fwd_kernel"


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


class Layer:
    """One layer of a step: its inputs, output buffer and launches."""

    def __init__(self, wl, x, dev, gdla=None):
        import torch
        self.wl = wl
        self.x = x
        n_tok = wl.B * wl.T
        self.kbuf = self.vbuf = None
        # the inputs a step brings from the host (decode: the query side; the
        # latent cache and W^KV_b stay resident)
        self.step_inputs = [n for n in x if not (wl.decode and n in ("c_kv", "w_kvb"))]
        # (label, kernel, flops, bytes, kernel launches) per library call
        self.launches = []
        if wl.decode:
            self.c_hat = gdla.gdla_latent_rmsnorm(x["c_kv"], None, wl.eps)
            self.cache_len = torch.full((wl.B,), wl.T, dtype=torch.int32, device=dev)
            self.ws = torch.empty(gdla.gdla_decode_workspace_bytes(wl.B, wl.T, wl.Hs, wl.Hn,
                                                                   wl.d_latent, wl.window),
                                  dtype=torch.uint8, device=dev)
            self.out = torch.empty((wl.B, wl.Hs * wl.d), dtype=torch.bfloat16, device=dev)
            # four kernels per call: absorb, attention, split merge, output GEMM
            self.launches.append(("%s/decode" % wl.name, "gdla_decode_attn_kernel",
                                  wl.attn_flops(), wl.decode_bytes(), 4))
            return
        if wl.bwd:
            # the six gradients in one buffer (the step's output), the scratch
            n_out = 0
            for sh in bwd_grad_shapes(wl).values():
                k = 1
                for e in sh:
                    k *= e
                n_out += k
            self.out = torch.empty(n_out, dtype=torch.bfloat16, device=dev)
            self.ws = torch.empty(gdla.gdla_attn_bwd_workspace_bytes(wl.B, wl.T, wl.Hs, wl.Hn,
                                                                     wl.d),
                                  dtype=torch.uint8, device=dev)
            self.launches.append(("%s/bwd" % wl.name, "gdla_attn_bwd", wl.bwd_flops(),
                                  wl.bwd_bytes(), 4))
            return
        if wl.latent:
            self.kbuf = torch.empty((n_tok, wl.Hkv, wl.d), dtype=torch.bfloat16, device=dev)
            self.vbuf = torch.empty_like(self.kbuf)
        self.out = torch.empty((wl.B, wl.T, wl.Hs * wl.d), dtype=torch.bfloat16, device=dev)
        if wl.latent:
            self.launches.append(("%s/expand" % wl.name, "gdla_kv_expand_kernel",
                                  wl.expand_flops(), wl.expand_bytes(), 1))
        self.launches.append(("%s/attn" % wl.name, attn_kernel_name(wl), wl.attn_flops(),
                              wl.attn_bytes(), 1))

    def run(self, gdla, status, stream, inp=None, out=None, events=None, cache_len=None):
        """Enqueue the layer; events[i] = (start, end) for launch i."""
        wl = self.wl
        inp = self.x if inp is None else inp
        out = self.out if out is None else out
        if wl.decode:
            if events is not None:
                events[0][0].record(stream)
            gdla.gdla_decode_fwd(inp["q_sig"], inp["q_noise"], self.c_hat,
                                 self.cache_len if cache_len is None else cache_len,
                                 self.x["w_kvb"], inp["lam"], inp["gate"], window=wl.window,
                                 out=out, workspace=self.ws, d_status=status, stream=stream)
            if events is not None:
                events[0][1].record(stream)
            return
        if wl.bwd:
            if events is not None:
                events[0][0].record(stream)
            gdla.gdla_attn_bwd(inp["q_sig"], inp["q_noise"], inp["k"], inp["v"], inp["lam"],
                               inp["gate"], inp["d_out"], window=wl.window, causal=wl.causal,
                               grads=bwd_grad_views(wl, out), workspace=self.ws,
                               d_status=status, stream=stream)
            if events is not None:
                events[0][1].record(stream)
            return
        li = 0
        if wl.latent:
            if events is not None:
                events[li][0].record(stream)
            gdla.gdla_kv_expand(inp["c_kv"], inp["w_kvb"], None, eps=wl.eps, d_head=wl.d,
                                k_out=self.kbuf, v_out=self.vbuf, d_status=status, stream=stream)
            if events is not None:
                events[li][1].record(stream)
            li += 1
            k = self.kbuf.view(wl.B, wl.T, wl.Hkv, wl.d)
            v = self.vbuf.view(wl.B, wl.T, wl.Hkv, wl.d)
        else:
            k, v = inp["k"], inp["v"]
        if events is not None:
            events[li][0].record(stream)
        if wl.d_rope:
            gdla.gdla_attn_fwd_rope(inp["q_sig"], inp["q_noise"], inp["q_rope_sig"],
                                    inp["q_rope_noise"], k, v, inp["k_rope"], inp["lam"],
                                    inp["gate"], window=wl.window, causal=wl.causal, out=out,
                                    d_status=status, stream=stream)
        else:
            gdla.gdla_attn_fwd(inp["q_sig"], inp["q_noise"], k, v, inp["lam"], inp["gate"],
                               window=wl.window, causal=wl.causal, out=out, d_status=status,
                               stream=stream)
        if events is not None:
            events[li][1].record(stream)


def _roofline_entry(label, kernel, flops, nbytes, avg_ms, peaks, peak_src, sustained,
                    traffic):
    """Roofline figures of one kernel launch (algorithmic work / event time)."""
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    tensor_bound = flops / max(1, nbytes) > ridge
    tflops = flops / (avg_ms * 1e-3) / 1e12
    gbs = nbytes / (avg_ms * 1e-3) / 1e9
    e = {"kernel": kernel, "launch": label, "avg_launch_ms": round(avg_ms, 4),
         "algorithmic_flop": flops, "algorithmic_bytes": nbytes,
         "tflops": round(tflops, 2), "gbs": round(gbs, 1)}
    if tensor_bound:
        burst = float(peaks["bf16_tflops"])
        sus = float(peaks["bf16_tflops_sustained"])
        peak = sus if sustained else burst
        e.update({"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                  "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                  "frac_of_burst": round(tflops / burst, 4),
                  "frac_of_sustained": round(tflops / sus, 4),
                  "peak_source": "%s %s" % (peak_src, "bf16_tflops_sustained" if sustained
                                            else "bf16_tflops")})
    else:
        peak = float(peaks["hbm_gbs"])
        e.update({"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                  "frac": round(gbs / peak, 4), "peak_source": "%s hbm_gbs" % peak_src})
    e["traffic"] = traffic
    return e


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
    layers = [Layer(WORKLOADS[n], make_inputs(WORKLOADS[n], seed=replica_seed(rank), device=dev),
                    dev, gdla) for n in STEPS[args.workload]]
    stream = torch.cuda.current_stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    n_launch = sum(len(L.launches) for L in layers)

    def step(events=None, inputs=None, outs=None, strm=None):
        st = stream if strm is None else strm
        li = 0
        for j, L in enumerate(layers):
            ev = None if events is None else events[li:li + len(L.launches)]
            L.run(gdla, status, st, inp=None if inputs is None else inputs[j],
                  out=None if outs is None else outs[j], events=ev)
            li += len(L.launches)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError("kernel reported status %d during warm-up" % int(status.item()))

    # decode steps are short enough for the host to fall behind the GPU, so
    # each library call is captured once in a CUDA graph and replayed (what a
    # serving loop does); the other steps launch eagerly
    graphs = None
    if not args.eager and all(L.wl.decode for L in layers):
        graphs = []
        for L in layers:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                L.run(gdla, status, torch.cuda.current_stream(dev))
            graphs.append(g)
        torch.cuda.synchronize(dev)

        def step(events=None, inputs=None, outs=None, strm=None):  # noqa: F811
            for j, g in enumerate(graphs):
                if events is not None:
                    events[j][0].record(stream)
                g.replay()
                if events is not None:
                    events[j][1].record(stream)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)

    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_launch)] for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(_gpu_id(torch, dev)) if rank == 0 else None
    time.sleep(0.25 if sampler else 0)
    if world > 1:
        dist.barrier()
    # a step that reads less than twice the L2 would run from L2 when repeated:
    # then the L2 is flushed (a buffer of twice its size written) before each
    # step, outside the step's own events, and the steps' times are summed
    l2_bytes = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or 126 << 20)
    step_bytes = sum(nb for L in layers for (_, _, _, nb, _) in L.launches)
    flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev) \
        if step_bytes < 2 * l2_bytes else None
    se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
            se[i][0].record(stream)
        step(events=ev[i])
        if flush is not None:
            se[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    ms = t0.elapsed_time(t1) if flush is None else \
        sum(a.elapsed_time(b) for (a, b) in se)
    launch_ms = [sum(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(args.steps)) /
                 args.steps for j in range(n_launch)]
    if int(status.item()) != 0:
        raise RuntimeError("kernel reported status %d" % int(status.item()))
    ms = max_over_ranks(ms, world, dev)
    # the first tokens of each output, for the parity figures of the CPU sample
    # (decode: every sequence's output over the first SAMPLE_SPAN cache rows)
    head_out = []
    for L in layers:
        if L.wl.decode:
            span = torch.full_like(L.cache_len, min(L.wl.T, SAMPLE_SPAN))
            o = torch.empty_like(L.out)
            L.run(gdla, status, stream, out=o, cache_len=span)
            head_out.append(o.float().cpu())
        elif L.wl.bwd:
            # the row-local gradients of the first BWD_SPAN tokens of batch 0
            gv = bwd_grad_views(L.wl, L.out)
            head_out.append({n: gv[n][:1, :min(L.wl.T, BWD_SPAN)].float().cpu()
                             for n in ("dq_sig", "dq_noise", "dlam", "dgate")})
        else:
            head_out.append(L.out[:1, :min(L.wl.T, SAMPLE_SPAN)].float().cpu())

    e2e_ms, e2e_steps, h2d, d2h = _e2e(args, layers, gdla, status, stream, dev, world)

    step_flops = sum(f for L in layers for (_, _, f, _, _) in L.launches)
    # tokens a step produces: every token of a prefill layer, one per sequence in decode
    n_tok = sum(L.wl.B * (1 if L.wl.decode else L.wl.T) for L in layers)
    value = step_flops * args.steps * world / (ms * 1e-3) / 1e12
    e2e_value = step_flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12
    peaks, peak_src = _peaks()
    sustained = ms * 1e-3 >= SUSTAINED_AFTER_S
    entries = []
    j = 0
    for L in layers:
        for (label, kernel, flops, nbytes, _) in L.launches:
            traffic = _traffic_from_profiles(L.wl.name, kernel)
            entries.append(_roofline_entry(label, kernel, flops, nbytes, launch_ms[j], peaks,
                                           peak_src, sustained, traffic))
            j += 1
    kernel_ms = sum(launch_ms)
    for e in entries:
        e["share_of_step"] = round(e["avg_launch_ms"] / (ms / args.steps), 4)
    top = max(entries, key=lambda e: e["avg_launch_ms"])
    wl0 = layers[0].wl
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
            "workload": args.workload,
            "layers": [{"name": L.wl.name, "B": L.wl.B, "T": L.wl.T, "window": L.wl.window,
                        "causal": L.wl.causal, "latent_kv": L.wl.latent or L.wl.decode,
                        "decode": L.wl.decode} for L in layers],
            "Hs": wl0.Hs, "Hn": wl0.Hn, "Hkv": wl0.Hkv, "d": wl0.d,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": ("inputs larger than L2 (%.0f MB per step)" % (step_bytes / 1e6))
            if flush is None else
            ("L2 flushed before each step (%.0f MB written; the step reads %.0f MB)"
             % (flush.numel() / 1e6, step_bytes / 1e6)),
            "launch": "CUDA graph per library call" if graphs is not None else "eager",
        },
        "roofline": top,
        "rooflines": entries,
        "kernel_ms_per_step": round(kernel_ms, 4),
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "mode": "pinned host buffers, eager library calls, copies pipelined per layer "
                        "with compute over 3 streams"},
        "gpu_launches": sum(k for L in layers for (_, _, _, _, k) in L.launches) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"], result["parity"] = cpu_baseline(layers, head_out,
                                                                seconds=args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def _e2e(args, layers, gdla, status, stream, dev, world):
    """End to end through the public API from pinned host memory: every step
    copies all its inputs host->device and its outputs device->host inside
    the timed region, and calls the library on them eagerly (no graph).  The
    copies are pipelined per layer over three streams with two device buffer
    sets (the resident inputs and outputs are the first set): the upload of
    a layer's next inputs and the download of its previous outputs overlap
    the kernels of the layers before it."""
    import torch
    import torch.distributed as dist

    long_step = any(L.wl.T >= 100000 for L in layers)
    e2e_steps = max(2, min(args.steps, 8 if long_step else 12))

    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    host = [{n: pinned_copy(L.x[n]) for n in L.step_inputs} for L in layers]
    out_host = [torch.empty(L.out.shape, dtype=L.out.dtype, pin_memory=True) for L in layers]
    h2d = sum(t.numel() * t.element_size() for hs in host for t in hs.values())
    d2h = sum(L.out.numel() * L.out.element_size() for L in layers)
    dev_in = [[L.x for L in layers], [dict(L.x, **{n: torch.empty_like(L.x[n])
                                                  for n in L.step_inputs}) for L in layers]]
    dev_out = [[L.out for L in layers], [torch.empty_like(L.out) for L in layers]]
    s_up, s_run, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    nl = len(layers)
    ev = {k: [[torch.cuda.Event() for _ in range(nl)] for _ in range(2)]
          for k in ("up", "run", "down")}
    for k in ev:
        for row in ev[k]:
            for e in row:
                e.record(stream)

    def e2e_step(i):
        b = i % 2
        for j in range(nl):
            s_up.wait_event(ev["run"][b][j])        # layer j's inputs of step i-2 consumed
            with torch.cuda.stream(s_up):
                for n, t in host[j].items():
                    dev_in[b][j][n].copy_(t, non_blocking=True)
                ev["up"][b][j].record(s_up)
        for j, L in enumerate(layers):
            s_run.wait_event(ev["up"][b][j])
            s_run.wait_event(ev["down"][b][j])      # layer j's outputs of step i-2 downloaded
            with torch.cuda.stream(s_run):
                L.run(gdla, status, s_run, inp=dev_in[b][j], out=dev_out[b][j])
                ev["run"][b][j].record(s_run)
            s_down.wait_event(ev["run"][b][j])
            with torch.cuda.stream(s_down):
                out_host[j].copy_(dev_out[b][j], non_blocking=True)
                ev["down"][b][j].record(s_down)

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
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if world > 1:
        dist.barrier()
    del host, out_host, dev_in, dev_out
    return e2e_ms, e2e_steps, h2d, d2h


def _strip_comments(src):
    """C/C++ source without its comments or blank-line differences."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


# The sources each kernel is built from (its launch code included): a
# profiled counter applies to a kernel only while these are unchanged.
KERNEL_SOURCES = {
    "gdla_attn_fwd_kernel": ("gdla_api.cu", "host_util.cuh", "attn_fwd.cuh", "sm100.cuh"),
    "gdla_attn_win_kernel": ("gdla_api.cu", "host_util.cuh", "attn_win.cuh", "attn_fwd.cuh",
                             "sm100.cuh"),
    "gdla_attn_rope_kernel": ("gdla_api.cu", "host_util.cuh", "attn_rope.cuh", "attn_win.cuh",
                              "attn_fwd.cuh", "sm100.cuh"),
    "gdla_kv_expand_kernel": ("gdla_api.cu", "host_util.cuh", "kv_expand.cuh", "sm100.cuh"),
    "gdla_decode_attn_kernel": ("gdla_api.cu", "host_util.cuh", "decode.cuh", "sm100.cuh"),
    "gdla_attn_bwd": ("gdla_bwd.cu", "host_util.cuh", "bwd.cuh", "attn_rope.cuh", "attn_win.cuh",
                      "attn_fwd.cuh", "sm100.cuh"),
}


def _csrc_hash(kernel=None):
    """Hash of the code (comments excluded) of the CUDA sources `kernel` is
    built from (every source when None), to tell whether profiled counters
    still apply to the kernel being timed."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "grouped_differential_attention_gdla_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel.split("<")[0]) if kernel else None
    files = [os.path.join(csrc, n) for n in names] if names else sorted(
        glob.glob(os.path.join(csrc, "*")))
    h = hashlib.sha256()
    for f in files:
        with open(f, encoding="utf-8") as fh:
            h.update(_strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def _traffic_from_profiles(name, kernel):
    """DRAM bytes (read + write) per launch of `kernel` on workload `name`
    from a committed ncu summary under profiles/ (a line "traffic:
    workload=<w> kernel=<k> csrc=<hash> bytes=<n>"), or None when none
    matches this workload, kernel and the kernel's current sources."""
    import glob
    kname = kernel.split("<")[0]
    want = _csrc_hash(kname)
    pat = re.compile(r"traffic: workload=(\S+) kernel=(\S+) csrc=(\S+) bytes=(\d+)")
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as f:
            for m in pat.finditer(f.read()):
                if m.group(1) == name and m.group(2) == kname and m.group(3) == want:
                    return int(m.group(4))
    return None


def _oracle_sample(wl, x, seconds, rng):
    """Time the float64 oracle on a bounded sample of one layer.

    Sample: query rows drawn uniformly from the first SAMPLE_SPAN tokens of
    batch element 0 (all heads), plus, for the latent layer, the RMSNorm +
    expand of those tokens.  Returns (flops, elapsed_s, description, rows,
    oracle outputs [n_rows, Hs*d]).
    """
    import numpy as np
    import torch

    import oracle

    span = min(wl.T, SAMPLE_SPAN)
    if wl.decode:
        return _oracle_decode_sample(wl, x, seconds, rng, span)
    if wl.bwd:
        return _oracle_bwd_sample(wl, x, seconds)
    # rows per pass: a sliding-window row costs W pairs, a causal row up to span
    n_rows = 256 if wl.window > 0 else 8
    total_flops, total_s = 0, 0.0
    cpu = {}
    for n in ("c_kv", "w_kvb", "k", "v", "k_rope"):
        if n in x:
            t = x[n]
            cpu[n] = (t[:span] if n == "c_kv" else
                      (t[:1, :span] if n in ("k", "v", "k_rope") else t)).cpu()
    all_rows, all_ref = [], []
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
        rope = {}
        if wl.d_rope:
            rope = dict(q_rope_sig_rows=g(x["q_rope_sig"]), q_rope_noise_rows=g(x["q_rope_noise"]),
                        k_rope=cpu["k_rope"])
        ref = oracle.gdla_attn_rows(g(x["q_sig"]), g(x["q_noise"]), k, v, g(x["lam"]),
                                    g(x["gate"]), rows, window=wl.window, causal=wl.causal, **rope)
        for i in rows:
            kept = min(int(i) + 1, wl.window) if wl.window > 0 else int(i) + 1
            flops += (4 * wl.d + 2 * wl.d_rope) * (wl.Hs + wl.Hn) * kept
        total_s += time.perf_counter() - t0
        total_flops += flops
        all_rows.append(rows)
        all_ref.append(ref)
    n_done = sum(len(r) for r in all_rows)
    desc = ("%s: %d query rows (all %d heads) drawn uniformly from the first %d tokens%s" % (
        wl.name, n_done, wl.Hs + wl.Hn, span,
        ", plus RMSNorm+W^KV_b expand of those %d tokens per pass" % span if wl.latent else ""))
    return total_flops, total_s, desc, np.concatenate(all_rows), np.concatenate(all_ref)


def _oracle_bwd_sample(wl, x, seconds):
    """The backward sample: the oracle's backward of the causal prefix of the
    first BWD_SPAN tokens of batch element 0, repeated for the time budget.
    Rows are token indices; ref holds the row-local gradients."""
    import oracle
    span = min(wl.T, BWD_SPAN)
    cpu = {n: x[n][:1, :span].cpu() for n in ("q_sig", "q_noise", "k", "v", "lam", "gate", "d_out")}
    sub = type(wl)(wl.name, B=1, T=span, Hs=wl.Hs, Hn=wl.Hn, Hkv=wl.Hkv, d=wl.d,
                   window=wl.window, causal=wl.causal, bwd=True)
    total_s, passes, ref = 0.0, 0, None
    while total_s < seconds or passes == 0:
        t0 = time.perf_counter()
        ref = oracle.gdla_attn_bwd(*(cpu[n] for n in ("q_sig", "q_noise", "k", "v", "lam", "gate",
                                                    "d_out")), window=wl.window,
                                   causal=wl.causal)
        total_s += time.perf_counter() - t0
        passes += 1
    desc = ("%s: the backward of the first %d tokens of batch element 0 (all %d heads), %d "
            "passes" % (wl.name, span, wl.Hs + wl.Hn, passes))
    return sub.bwd_flops() * passes, total_s, desc, None, ref


def _oracle_decode_sample(wl, x, seconds, rng, span):
    """The decode sample: sequences drawn uniformly, each decoding its token
    at cache length `span` (RMSNorm + expand of the kept cache rows and the
    forward pass for the one query row).  Rows are sequence indices."""
    import numpy as np

    import oracle

    n_seq = 16 if wl.window > 0 else 1
    total_flops, total_s = 0, 0.0
    all_rows, all_ref = [], []
    w = x["w_kvb"].cpu()
    while total_s < seconds:
        rows = np.sort(rng.integers(0, x["q_sig"].shape[0], n_seq))
        t0 = time.perf_counter()
        sub = {n: x[n][rows].cpu() for n in ("q_sig", "q_noise", "lam", "gate")}
        c = x["c_kv"][rows, :span].cpu()
        ref = oracle.decode(sub["q_sig"], sub["q_noise"], c, [span] * n_seq, w, sub["lam"],
                            sub["gate"], eps=wl.eps, window=wl.window)
        total_s += time.perf_counter() - t0
        kept = min(span, wl.window) if wl.window > 0 else span
        total_flops += n_seq * 4 * wl.d * (wl.Hs + wl.Hn) * kept
        all_rows.append(rows)
        all_ref.append(ref)
    n_done = sum(len(r) for r in all_rows)
    desc = ("%s: %d sequences drawn uniformly, each decoding at cache length %d (RMSNorm + "
            "W^KV_b expand of the kept cache rows, then the forward pass of the query token)" % (
                wl.name, n_done, span))
    return total_flops, total_s, desc, np.concatenate(all_rows), np.concatenate(all_ref)


def _parity(gpu_rows, ref):
    """Error statistics of GPU output rows against the oracle's (per tensor
    tolerance max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3)."""
    import numpy as np
    diff = np.abs(gpu_rows - ref)
    idx = np.unravel_index(int(np.argmax(diff)), diff.shape)
    max_ref = float(np.abs(ref).max())
    tol = 1e-2 * max_ref + 1e-3
    return {"rows": int(ref.shape[0]), "max_abs_err": float(diff.max()),
            "mean_abs_err": float(diff.mean()), "rms_err": float(np.sqrt((diff ** 2).mean())),
            "max_abs_oracle": max_ref, "tol": tol, "pass": bool(diff.max() <= tol),
            "argmax_sample_col": [int(idx[0]), int(idx[1])]}


def cpu_baseline(layers, head_out, seconds=15.0):
    """The oracle timed on host cores over a bounded sample of every layer of
    the step, and the parity figures of the GPU output on the same rows."""
    import numpy as np
    rng = np.random.default_rng(0)
    flops, secs, descs, parity = 0, 0.0, [], {}
    for L, ho in zip(layers, head_out):
        f, s, d, rows, ref = _oracle_sample(L.wl, L.x, seconds / len(layers), rng)
        flops += f
        secs += s
        descs.append(d)
        if L.wl.bwd:
            for n, g in ho.items():
                span = g.shape[1]
                parity["%s/%s" % (L.wl.name, n)] = _parity(
                    g[0].reshape(span, -1).numpy().astype(np.float64),
                    ref[n][0].reshape(span, -1))
            continue
        gpu_rows = (ho if L.wl.decode else ho[0]).numpy()[rows].astype(np.float64)
        parity[L.wl.name] = _parity(gpu_rows, ref)
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return ({"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
             "kind": "oracle", "sample": "; ".join(descs) + " (float64 oracle)",
             "seconds": round(secs, 2)}, parity)


def run_reference(args):
    """Reference arm: the float64 CPU oracle on a bounded sample per step."""
    world, rank, local = _dist()
    if rank != 0:
        return
    import numpy as np

    from grouped_differential_attention_gdla_b200.inputs import WORKLOADS, make_inputs
    import oracle

    oracle.build()
    wls = [WORKLOADS[n] for n in STEPS[args.workload]]
    # inputs drawn on the CPU in the same recipe; only the sampled slices are used
    xs = [make_inputs(wl, seed=0, device="cpu", T=min(wl.T, SAMPLE_SPAN),
                      B=(min(wl.B, 16) if wl.decode else 1)) for wl in wls]
    per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        for wl, x in zip(wls, xs):
            _oracle_sample(wl, x, per_step / 4 / len(wls), rng)
    flops, secs = 0, 0.0
    descs = []
    for _ in range(args.steps):
        descs = []
        for wl, x in zip(wls, xs):
            f, s, d, _, _ = _oracle_sample(wl, x, per_step / len(wls), rng)
            flops += f
            secs += s
            descs.append(d)
    value = flops / secs / 1e12
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    n_tok = sum(wl.B * (1 if wl.decode else wl.T) for wl in wls)
    step_flops = sum(wl.attn_flops() + (wl.expand_flops() if wl.latent else 0) for wl in wls)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3 / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same recipe, CPU draw)",
        "config": {"workload": args.workload,
                   "layers": [{"name": wl.name, "B": wl.B, "T": wl.T, "window": wl.window,
                               "causal": wl.causal, "latent_kv": wl.latent or wl.decode,
                               "decode": wl.decode} for wl in wls],
                   "Hs": wls[0].Hs, "Hn": wls[0].Hn, "Hkv": wls[0].Hkv, "d": wls[0].d},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": "; ".join(descs) + " (per step)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
        "note": "float64 CPU oracle on %d host threads; tokens/s of the full workload would be "
                "%.3g" % (threads, n_tok * value * 1e12 / max(1, step_flops)),
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long", choices=sorted(STEPS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=16.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch decode steps eagerly instead of replaying CUDA graphs")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
