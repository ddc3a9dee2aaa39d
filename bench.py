#!/usr/bin/env python
"""Throughput of the quantised-base + LoRA linear on B200: fwd+bwd tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload lqlora|qalora|tiny|mlp7b|decode70b|lqlora_init]
                    [--impl ours|reference] [--no-extra] [--no-cpu-baseline]

One step = forward (adapter down-projection T = s P(X) A^T, fused dequant + tcgen05 base GEMM with the
adapter term folded in) + backward (dT, dA, dB; fused input gradient) of every linear of the workload,
over one batch of synthetic tokens already resident in HBM.  The default workload is the largest one that
fits one GPU: the 32-layer LLaMA-7B-shaped stack of 224 linears with per-matrix NF-k bit widths (2, 3, 4)
and blocks (64, 128) drawn from the seed, r = 64, 2048 tokens; every linear has its own activations X and
output gradients dY.  The same JSON line carries the QA-LoRA layer, the LLaMA-7B MLP block and the
decode-shape projection as extra keys (N = 1 only).  Rank 0 prints one JSON line.

Under torchrun (N > 1) every rank runs the workload on its own tokens (data parallel, weights replicated)
and the adapter gradients are summed over ranks with NCCL each step; the time is the maximum over ranks.
`--impl reference` times the CPU oracle (test infrastructure) on rank 0 only.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd tokens/s through quant-base+LoRA linears; % of TC peak / HBM GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="lqlora",
                    choices=["qalora", "tiny", "mlp7b", "lqlora", "decode70b", "lqlora_init"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' legs")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------ accounting
def flush_l2(buf, lead_ms: float = 1.0):
    """Evict the step's data from L2: write a buffer larger than L2, then read it back, so that the
    timed step neither hits in L2 nor pays for writing back the flush's own dirty lines.  First the stream
    spins for `lead_ms` on the device, so that the host enqueues the flush, the start event and the whole
    timed step while the GPU is still busy: the events then time the GPU's work, with no gaps where it
    waits for the host to launch the next kernel (the small workloads launch faster than Python can)."""
    import torch
    if lead_ms > 0:
        torch.cuda._sleep(int(lead_ms * 2.0e6))  # ~2e6 SM cycles per ms at the B200's clocks
    buf.zero_()
    return buf.view(torch.int32).amax()


def time_quantizer(qlr, spec, W, flush, reps: int = 10):
    """HBM roofline of the layer's own quantisation (the memory-bound quantiser path): median CUDA-event
    time of quantising the fp32 weight W already on the device, and its algorithmic bytes (fp32 read,
    codes and constants written)."""
    import torch
    N, K = spec.N, spec.K
    if spec.fmt == "int4g":
        fn = lambda: qlr.quantize_int4_group(W, spec.group)  # noqa: E731
        out_b = N * K // 2 + 4 * N * K // spec.group
        kern = f"quantize_int4g_kernel<{spec.group}>"
    else:
        fn = lambda: qlr.quantize_nf4(W, spec.bits, spec.block, spec.dq_block)  # noqa: E731
        nb = N * K // spec.block
        out_b = N * K * spec.bits // 8 + (nb + 4 * (nb // 256) if spec.dq_block else 4 * nb)
        kern = "quantize_nfk_kernel"
    for _ in range(2):
        fn()
    ts = []
    for _ in range(reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ts)
    nbytes = 4 * N * K + out_b
    return {"kernel": kern, "shape": [N, K], "ms": ms, "bytes": nbytes, "GBps": nbytes / ms / 1e6}


def flops_per_token(spec) -> float:
    """4NK (forward base GEMM + input gradient; the base weight gets no gradient) plus the six rank-r
    adapter products (T, T B^T, dT, dT A, dA, dB), with K/L adapter inputs for the pooled adapter."""
    ka = spec.k_adapter
    return 4.0 * spec.N * spec.K + 2.0 * spec.r * (3 * spec.N + 3 * ka)


def workload_desc(wl):
    spec = wl.linears[0]
    if wl.name == "qalora":
        return (f"qalora: INT4 group-{spec.group} base {spec.N}x{spec.K}, pooled adapter r={spec.r} "
                f"(s={spec.s}), {wl.M} tokens, fwd+bwd")
    if wl.name == "mlp7b":
        return f"mlp7b: LLaMA-7B MLP (gate/up 11008x4096, down 4096x11008) NF4+DQ, r=64, SwiGLU, {wl.M} tokens, fwd+bwd"
    if wl.name == "lqlora":
        return (f"lqlora: 32-layer LLaMA-7B stack, 224 linears (q,k,v,o 4096x4096; gate,up 11008x4096; "
                f"down 4096x11008), per-matrix NF-k (k in 2,3,4) and block (64/128) with double quantisation, "
                f"r=64, {wl.M} tokens, fwd+bwd")
    return f"tiny: NF4+DQ 256x256, r=8, {wl.M} tokens, fwd+bwd"


FUSED_SOURCES = ("fused.cu", "engine.cuh", "ptx.cuh", "gemm.cuh")


def fused_source_sha256() -> str:
    dig = hashlib.sha256()
    for f in FUSED_SOURCES:
        dig.update(open(os.path.join(ROOT, "quantized_base_lora_nf4_b200", "csrc", f), "rb").read())
    return dig.hexdigest()


def profile_traffic(keys):
    """Per-launch DRAM bytes (read + write) of the fused kernel launches named by `keys`, from the committed
    machine-readable capture profiles/fused_traffic.json, averaged over the keys; None unless every key was
    captured and the capture was taken on the current source of the fused kernel."""
    p = os.path.join(ROOT, "profiles", "fused_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("fused_source_sha256") != fused_source_sha256():
        return None
    per = d.get("bytes_per_launch", {})
    vals = [per.get(k) for k in keys]
    if not vals or any(v is None for v in vals):
        return None
    return float(sum(vals) / len(vals))


def traffic_key(kind: str, spec, M: int) -> str:
    """Key of one fused launch in profiles/fused_traffic.json: direction, shape, format, tokens."""
    fmt = f"nf{spec.bits}b{spec.block}" if spec.fmt == "nfk" else f"int4g{spec.group}"
    return f"{kind}:{spec.N}x{spec.K}:{fmt}:r{spec.r}:M{M}"


# ------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------ GPU arm
class Layer:
    """Device-resident state of one quantised linear: its weight, adapters, activations and gradients.

    With `on_device` (the mixed-precision stack) every tensor is drawn on the device with torch's seeded
    CUDA generator (the same laws as the numpy generators: W ~ N(0, sigma_W^2), A, B ~ N(0, 0.01^2), X and dY
    ~ N(0, 1)), which keeps the setup of 224 7B-sized linears short.  Every linear owns its X, dY, Y, dX,
    T and dT, so no linear finds another's activations in L2."""

    def __init__(self, qlr, spec, M, seed, rank, dev, X=None, on_device=False):
        import numpy as np
        import torch
        from synth import normal

        self.spec = spec
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16).contiguous()  # noqa
        r = spec.r
        if on_device:
            g = torch.Generator(device=dev)
            g.manual_seed(seed)
            W = torch.randn((spec.N, spec.K), generator=g, device=dev, dtype=torch.float32) * spec.sigma_w
            self.A = (torch.randn((r, spec.k_adapter), generator=g, device=dev) * 0.01).to(torch.bfloat16)
            self.B = (torch.randn((spec.N, r), generator=g, device=dev) * 0.01).to(torch.bfloat16)
            gr = torch.Generator(device=dev)
            gr.manual_seed(seed * 1009 + 17 * rank + 1)
            self.X = X if X is not None else torch.randn((M, spec.K), generator=gr, device=dev).to(torch.bfloat16)
            self.dY = torch.randn((M, spec.N), generator=gr, device=dev).to(torch.bfloat16)
        else:  # the seeded numpy streams the tests use; weights and adapters replicated, tokens per rank
            W = torch.from_numpy(normal(seed, 0, "W", (spec.N, spec.K), spec.sigma_w, bf16=False)).to(dev)
            self.A = bf(normal(seed, 0, "A", (r, spec.k_adapter), 0.01, bf16=True))
            self.B = bf(normal(seed, 0, "B", (spec.N, r), 0.01, bf16=True))
            self.X = X if X is not None else bf(normal(seed + 1000 * rank, 0, "X", (M, spec.K), 1.0, bf16=True))
            self.dY = bf(normal(seed + 1000 * rank, 0, "dY", (M, spec.N), 1.0, bf16=True))
        if spec.fmt == "int4g":
            self.q = qlr.quantize_int4_group(W, spec.group)
        else:
            self.q = qlr.quantize_nf4(W, spec.bits, spec.block, spec.dq_block)
        del W
        e = lambda shape, dt=torch.bfloat16: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
        self.T, self.dT = e((M, r)), e((M, r))
        self.Y, self.dX = e((M, spec.N)), e((M, spec.K))
        self.dA = e((r, spec.k_adapter), torch.float32)
        self.dB = e((spec.N, r), torch.float32)
        self.ws, self.ws_b, self.ws_x = qlr.Workspace(dev), qlr.Workspace(dev), qlr.Workspace(dev)
        self.ws_s = qlr.Workspace(dev)  # the adapter gradients' second stream


def run_ours(args, wl_name, rank, world, dev, steps, warmup, e2e_steps=None, swiglu_fused=False):
    """Times `steps` training steps of workload `wl_name` (after `warmup` untimed ones) with CUDA events on
    the stream the kernels run on, L2 flushed before each step; then the same step end to end from pinned
    host memory.  Returns the measurements (time is the max over ranks)."""
    import torch
    import torch.distributed as dist
    from quantized_base_lora_nf4_b200 import dp, qlr
    from synth import workload

    qlr.lib()
    wl = workload(wl_name, args.seed)
    M = wl.M
    seed = args.seed
    Hm = dHm = dG = dU = None
    if wl.kind == "mlp":
        gate_s, up_s, down_s = wl.linears
        gate = Layer(qlr, gate_s, M, seed, rank, dev)
        up = Layer(qlr, up_s, M, seed + 1, rank, dev, X=gate.X)
        Hm = torch.empty((M, gate_s.N), dtype=torch.bfloat16, device=dev)
        down = Layer(qlr, down_s, M, seed + 2, rank, dev, X=Hm)
        layers = [gate, up, down]
        dHm, dG, dU = torch.empty_like(Hm), torch.empty_like(Hm), torch.empty_like(Hm)
    elif wl.kind == "stack":
        layers = [Layer(qlr, spec, M, seed * 100003 + i, rank, dev, on_device=True) for i, spec in enumerate(wl.linears)]
        torch.cuda.synchronize()
    else:
        layers = [Layer(qlr, wl.linears[0], M, seed, rank, dev)]
    fwd_ev, dx_ev = [], []

    def timed(record, sink, fn):
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            sink.append((e0, e1))
        else:
            fn()

    def fwd_base(L, record, X=None):
        timed(record, fwd_ev, lambda: qlr.forward_base(L.q, L.X if X is None else X, L.B, L.T, Y=L.Y))

    # The adapter gradients dB and dA are needed by nothing else in the step, so they run on a second stream
    # that waits for dT, beside the input gradient on the main stream (which also waits only for dT).
    main_s = torch.cuda.current_stream()
    side = torch.cuda.Stream()

    def adapter_bwd(L, dY, X=None):
        """dT on the main stream; dB, dA on the side stream once dT is written."""
        qlr.backward_lora_dT(L.q, dY, L.B, L.spec.s, dT=L.dT, ws=L.ws_b)
        ev = torch.cuda.Event()
        ev.record(main_s)
        side.wait_event(ev)
        qlr.backward_lora_dAdB(L.q, L.X if X is None else X, dY, L.T, L.dT, pooled=L.spec.pooled, dA=L.dA, dB=L.dB,
                               ws=L.ws_s, stream=side)

    def lin_bwd(L, dY, dX, record, accumulate=False):
        adapter_bwd(L, dY)
        timed(record, dx_ev, lambda: qlr.backward_dx(L.q, dY, L.A, L.dT, pooled=L.spec.pooled, dX=dX,
                                                     accumulate=accumulate, ws=L.ws_x))

    # data parallel: the adapter gradients are summed over ranks.  A stack's linears are exchanged in
    # buckets whose all-reduce starts as soon as the last linear in them has finished its backward, so
    # the exchange overlaps the backward of the linears after it; a single linear or an MLP block is
    # one bucket, started when its backward ends
    buckets = None
    if world > 1:
        if wl.kind == "stack":
            buckets = dp.OverlappedBuckets([[L.dA, L.dB] for L in layers])
        else:
            buckets = dp.OverlappedBuckets([[g for L in layers for g in (L.dA, L.dB)]])

    def step(record=False):
        if wl.kind == "mlp":
            gate, up, down = layers
            qlr.lora_down(gate.q, gate.X, gate.A, gate.spec.s, T_save=gate.T, ws=gate.ws)
            qlr.lora_down(up.q, up.X, up.A, up.spec.s, T_save=up.T, ws=up.ws)
            fwd_base(gate, record)
            if swiglu_fused:  # the up projection with the SwiGLU gate in its epilogue: U and H in one launch
                timed(record, fwd_ev, lambda: qlr.forward_swiglu(up.q, up.X, up.B, up.T, gate.Y, U=up.Y, H=Hm))
            else:
                fwd_base(up, record)
                qlr.swiglu_forward(gate.Y, up.Y, H=Hm)
            qlr.lora_down(down.q, Hm, down.A, down.spec.s, T_save=down.T, ws=down.ws)
            fwd_base(down, record)
            adapter_bwd(down, down.dY, X=Hm)
            if swiglu_fused:  # the down projection's input gradient dH turned into (dG, dU) in its epilogue
                timed(record, dx_ev, lambda: qlr.backward_dx_swiglu(down.q, down.dY, down.A, down.dT, gate.Y, up.Y,
                                                                    dG=dG, dU=dU))
            else:
                timed(record, dx_ev, lambda: qlr.backward_dx(down.q, down.dY, down.A, down.dT, dX=dHm, ws=down.ws_x))
                qlr.swiglu_backward(dHm, gate.Y, up.Y, dG=dG, dU=dU)
            lin_bwd(gate, dG, gate.dX, record)
            lin_bwd(up, dU, gate.dX, record, accumulate=True)
        else:  # one linear, or every linear of the stack in turn
            for i, L in enumerate(layers):
                qlr.lora_down(L.q, L.X, L.A, L.spec.s, pooled=L.spec.pooled, T_save=L.T, ws=L.ws)
                fwd_base(L, record)
                lin_bwd(L, L.dY, L.dX, record)
                if buckets is not None and wl.kind == "stack":
                    buckets.layer_done(i, stream=side)
        if buckets is not None:
            if wl.kind != "stack":
                buckets.layer_done(0, stream=side)
            buckets.finish()
        main_s.wait_stream(side)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    launches0 = qlr.launch_count()
    evs = []
    for _ in range(steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step()  # no events inside: one recorded between two launches keeps the second from starting early
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize()
    launches = qlr.launch_count() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    # the fused kernels' own durations (roofline, step breakdown): the same number of steps again, each fused
    # launch between an event pair on its stream
    for _ in range(steps):
        flush_l2(flush)
        step(record=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms_steps = [a.elapsed_time(b) for a, b in evs]
    ms_total = sum(ms_steps)
    fwd_ms = [a.elapsed_time(b) for a, b in fwd_ev]
    dx_ms = [a.elapsed_time(b) for a, b in dx_ev]
    if world > 1:
        t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_per_step = ms_total / steps

    # end to end: the step's inputs (the first linear's activations and the last linear's output gradient,
    # as a training step receives them: the stack's inner activations stand for tensors a model produces
    # on the device) copied from pinned host memory every step, and its result (the last linear's adapter
    # gradients; every adapter gradient of a single linear or block) read back
    first, last = layers[0], layers[-1]
    h_in = [(first, "X", torch.empty(first.X.shape, dtype=torch.bfloat16, pin_memory=True)),
            (last, "dY", torch.empty(last.dY.shape, dtype=torch.bfloat16, pin_memory=True))]
    for L, a, h in h_in:
        h.copy_(getattr(L, a))
    out_layers = layers[-1:] if wl.kind == "stack" else layers
    h_out = [(L.dA, torch.empty(L.dA.shape, dtype=torch.float32, pin_memory=True)) for L in out_layers]
    h_out += [(L.dB, torch.empty(L.dB.shape, dtype=torch.float32, pin_memory=True)) for L in out_layers]
    h2d = sum(h.numel() * h.element_size() for _, _, h in h_in)
    d2h = sum(h.numel() * h.element_size() for _, h in h_out)
    n_e2e = e2e_steps if e2e_steps is not None else max(3, steps // 2)
    # inputs double-buffered: step i + 1's host-to-device copy runs on a copy stream while step i computes,
    # as a data loader would; each step still copies its inputs in and reads its result back
    inputs = []
    for L, a, h in h_in:
        d = getattr(L, a)
        refs = [(LL, aa) for LL in layers for aa in ("X", "dY") if getattr(LL, aa) is d]
        inputs.append((h, [d, torch.empty_like(d)], refs))

    def bind(slot):
        for _, bufs, refs in inputs:
            for LL, aa in refs:
                setattr(LL, aa, bufs[slot])

    copy_stream = torch.cuda.Stream()

    def run_e2e(n, start_event=None):
        ev_copy = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        with torch.cuda.stream(copy_stream):
            if start_event is not None:
                copy_stream.wait_event(start_event)
            for h, bufs, _ in inputs:
                bufs[0].copy_(h, non_blocking=True)
            ev_copy[0].record(copy_stream)
        for i in range(n):
            if i + 1 < n:
                with torch.cuda.stream(copy_stream):
                    if i >= 1:
                        copy_stream.wait_event(ev_done[i - 1])  # the buffer was last read by step i - 1
                    for h, bufs, _ in inputs:
                        bufs[(i + 1) % 2].copy_(h, non_blocking=True)
                    ev_copy[i + 1].record(copy_stream)
            main_s.wait_event(ev_copy[i])
            bind(i % 2)
            step()
            for d, h in h_out:
                h.copy_(d, non_blocking=True)
            ev_done[i].record(main_s)
        bind(0)

    run_e2e(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_s.record()
    run_e2e(n_e2e, start_event=e_s)
    e_e.record()
    torch.cuda.synchronize()
    e2e_ms = e_s.elapsed_time(e_e)
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    if world > 1:
        dist.barrier()
    res = {"wl": wl, "M": M, "steps": steps, "ms_per_step": ms_per_step, "ms_steps": ms_steps, "fwd_ms": fwd_ms,
           "dx_ms": dx_ms, "launches": launches, "clocks": clk, "e2e_ms_per_step": e2e_ms / n_e2e, "h2d": h2d,
           "d2h": d2h}
    del layers, flush
    torch.cuda.empty_cache()
    return res


def summarize(res, world, peaks, peak_kind):
    """Throughput, tensor-core fractions and the fused forward's roofline of one workload's run."""
    wl, M, ms = res["wl"], res["M"], res["ms_per_step"]
    fl_tok = sum(flops_per_token(s) for s in wl.linears)
    peak = float(peaks["bf16_tflops"])
    tflops = world * fl_tok * M / (ms / 1e3) / 1e12
    n_lin = len(wl.linears)
    steps = res["steps"]
    fwd_ms, dx_ms = res["fwd_ms"], res["dx_ms"]
    fwd_fl = [2.0 * M * s.N * (s.K + s.r) for s in wl.linears]
    dx_fl = [2.0 * M * s.K * (s.N + s.r) for s in wl.linears]
    # per linear, mean over the timed steps (events are recorded in step order, one per linear)
    fwd_per = [statistics.mean(fwd_ms[i::n_lin]) for i in range(n_lin)]
    dx_per = [statistics.mean(dx_ms[i::n_lin]) for i in range(n_lin)]
    fwd_launch_ms = sum(fwd_per) / n_lin
    fwd_flops = sum(fwd_fl) / n_lin
    achieved = fwd_flops / (fwd_launch_ms / 1e3) / 1e12
    traffic = profile_traffic([traffic_key("fwd", s, M) for s in wl.linears])
    step_fwd, step_dx = sum(fwd_per), sum(dx_per)
    out = {
        "value": world * M / (ms / 1e3), "ms_per_step": ms, "tflops": tflops,
        "tc_frac_of_measured_burst": tflops / peak,
        "tc_frac_of_measured_sustained": tflops / float(peaks.get("bf16_tflops_sustained", peak)),
        "roofline": {"bound": "tensor", "kernel": "fused_kernel<A_DQ_K> (fused dequant + tcgen05 forward)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16 burst", "traffic": traffic,
                     "flops_per_launch": fwd_flops, "launch_ms": fwd_launch_ms,
                     "launches_averaged": n_lin},
        "step_breakdown_ms": {
            "fused_forward": step_fwd, "fused_input_gradient": step_dx,
            "adapter_and_rest": ms - step_fwd - step_dx,
            "fused_forward_TFLOPs": sum(fwd_fl) / (step_fwd / 1e3) / 1e12,
            "fused_input_gradient_TFLOPs": sum(dx_fl) / (step_dx / 1e3) / 1e12,
            # per launch, in launch order (the MLP block's input gradients run down, gate, up)
            **({"fused_forward_per_launch": fwd_per, "fused_input_gradient_per_launch": dx_per} if n_lin <= 8 else {})},
        "gpu_launches": res["launches"], "gpu_launches_per_step": res["launches"] / steps,
        "clocks": res["clocks"],
        "e2e": {"value": world * M / (res["e2e_ms_per_step"] / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                "ms_per_step": res["e2e_ms_per_step"],
                "pipeline": "pinned host inputs (the first linear's X, the last linear's dY) copied in every step, "
                            "double-buffered on a copy stream so that step i+1's copy overlaps step i's compute; "
                            "the step's adapter gradients (the stack: the last linear's) read back"},
    }
    return out


# ------------------------------------------------------------------------------------------ CPU oracle arm
def oracle_tokens_per_s(wl, seed, budget_s=10.0):
    """Times the oracle (test infrastructure, as it stands) on the host cores on a bounded sample of the
    workload: the oracle's quantiser once per sampled linear (timed, reported apart: a training step does not
    quantise), then forward + backward of `m` tokens through the sampled linears with fp32 contractions
    (numpy BLAS) on the dequantised weights, repeated for about `budget_s`.  The stack is sampled by the
    first linear of each of its three shapes, and its rate scaled by FLOPs to all 224 linears."""
    import numpy as np
    from oracle import layer as OL
    from oracle import quantize as Q
    from synth import linear_tensors

    m = {"tiny": 16, "qalora": 2048, "mlp7b": 1024, "lqlora": 2048}[wl.name]
    linears = list(wl.linears)
    scale = 1.0
    if wl.kind == "stack":
        seen, sample = set(), []
        for spec in linears:
            if (spec.N, spec.K) not in seen:
                seen.add((spec.N, spec.K))
                sample.append(spec)
        scale = sum(flops_per_token(s) for s in sample) / sum(flops_per_token(s) for s in linears)
        linears = sample
    f32 = np.float32
    mats, quant_s = [], {}
    for i, spec in enumerate(linears):
        t = linear_tensors(spec, m, seed=seed + i)
        t0 = time.perf_counter()
        if spec.fmt == "int4g":
            Wdq = Q.dequant_int4_group(Q.quantize_int4_group(t["W"], spec.group))
        else:
            Wdq = Q.dequant_nfk(Q.quantize_nfk(t["W"], spec.bits, spec.block, spec.dq_block))
        quant_s[f"{spec.name} {spec.N}x{spec.K}"] = time.perf_counter() - t0
        mats.append((spec, t, Wdq.astype(f32)))
    reps, t0 = 0, time.perf_counter()
    while True:
        if wl.kind == "mlp":
            (gs, gt, gW), (us, ut, uW), (ds, dt, dW) = mats
            X = gt["X"]
            G = OL.forward(X, gW, gt["A"], gt["B"], gs.s, dtype=f32)["Y"]
            U = OL.forward(X, uW, ut["A"], ut["B"], us.s, dtype=f32)["Y"]
            Hm = OL.swiglu_forward(G, U).astype(f32)
            OL.forward(Hm, dW, dt["A"], dt["B"], ds.s, dtype=f32)
            bd = OL.backward(dt["dY"], Hm, dW, dt["A"], dt["B"], ds.s, dtype=f32)
            dG, dU = OL.swiglu_backward(bd["dX"], G, U)
            OL.backward(dG, X, gW, gt["A"], gt["B"], gs.s, dtype=f32)
            OL.backward(dU, X, uW, ut["A"], ut["B"], us.s, dtype=f32)
        else:
            for spec, t, Wdq in mats:
                L = spec.group if spec.pooled else None
                OL.forward(t["X"], Wdq, t["A"], t["B"], spec.s, L, dtype=f32)
                OL.backward(t["dY"], t["X"], Wdq, t["A"], t["B"], spec.s, L, dtype=f32)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 2000:
            break
    cores = len(os.sched_getaffinity(0))
    what = (f"{reps} x {m} tokens through the first linear of each of the {len(mats)} shapes of the stack, "
            f"scaled by FLOPs (x{scale:.4f}) to all {len(wl.linears)} linears" if wl.kind == "stack"
            else f"{reps} x {m} tokens of the {wl.name} workload")
    return {"value": reps * m / el * scale, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{what}: fwd+bwd with fp32 numpy BLAS contractions ({el:.1f} s); the oracle's quantiser "
                      f"timed once per sampled linear ({sum(quant_s.values()):.1f} s)",
            "quantize_s": quant_s, "contractions": "fp32"}


# ------------------------------------------------------------------------------------------ LQ-LoRA init
def run_lqlora_init(args, dev, iters: int = 2):
    """LQ-LoRA initialisation (alternating rank-64 SVD of the residual and NF-k quantisation) of the first
    matrix of each distinct shape of the 7B stack, with its drawn bit width and block; CUDA-event time of
    the whole call (the SVD is cuSOLVER's), projected to the stack's 224 matrices."""
    import torch
    from quantized_base_lora_nf4_b200 import qlr
    from synth import workload

    wl = workload("lqlora", args.seed)
    seen, out = {}, {}
    for spec in wl.linears:
        if (spec.N, spec.K) in seen:
            continue
        g = torch.Generator(device=dev)
        g.manual_seed(args.seed)
        W = torch.randn((spec.N, spec.K), generator=g, device=dev, dtype=torch.float32) * spec.sigma_w
        qlr.lqlora_init(W, spec.bits, spec.block, spec.dq_block, spec.r, spec.s, iters)  # warm-up (solver load)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qlr.lqlora_init(W, spec.bits, spec.block, spec.dq_block, spec.r, spec.s, iters)
        e1.record()
        torch.cuda.synchronize()
        seen[(spec.N, spec.K)] = e0.elapsed_time(e1)
        out[f"{spec.N}x{spec.K}"] = {"ms": seen[(spec.N, spec.K)], "bits": spec.bits, "block": spec.block,
                                     "r": spec.r, "iters": iters}
        del W
    stack_s = sum(seen[(s_.N, s_.K)] for s_ in wl.linears) / 1e3
    alloc = run_lqlora_allocation(args, dev, wl)
    return {"metric": "LQ-LoRA initialisation time per matrix (ms), whole call", "per_shape": out,
            "stack_projection_s": stack_s, "stack_matrices": len(wl.linears), "allocation": alloc,
            "note": "truncated SVD: top-r eigenpairs of the smaller-side Gram matrix (fp32 cuBLAS syrk + "
                    "cuSOLVER syevdx) and one projection GEMM; residual, rank-r subtraction, factor split and "
                    "quantisation in this library's kernels"}


def run_lqlora_allocation(args, dev, wl):
    """Budgeted (bits, block) plan for the 224 matrices of the 7B stack: the quantisation error of all six
    options of every matrix on the GPU, then the library's exact allocation at the storage budget of the
    stack's seeded per-matrix draw; reports both plans' total errors."""
    import numpy as np
    import torch
    from quantized_base_lora_nf4_b200 import qlr

    L = qlr.lib()
    options = [(k, b) for k in (2, 3, 4) for b in (64, 128)]
    m = len(wl.linears)
    err = np.zeros((m, len(options)))
    cost = np.zeros((m, len(options)), dtype=np.int64)
    drawn = []
    out = torch.empty((m, len(options)), dtype=torch.float64, device=dev)
    ws = None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_ms = 0.0
    for i, spec in enumerate(wl.linears):
        g = torch.Generator(device=dev)
        g.manual_seed(args.seed * 100003 + i)
        W = torch.randn((spec.N, spec.K), generator=g, device=dev, dtype=torch.float32) * spec.sigma_w
        nbytes = max(int(L.qlr_nf_quant_error_workspace_bytes(spec.N, spec.K, k, b, 256)) for k, b in options)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        e0.record()
        for o, (k, b) in enumerate(options):
            qlr.nf_quant_error(W, k, b, 256, out=out[i, o:o + 1], ws=ws)
        e1.record()
        torch.cuda.synchronize()
        gpu_ms += e0.elapsed_time(e1)
        for o, (k, b) in enumerate(options):
            cost[i, o] = 8 * sum(qlr.part_bytes(qlr.FMT_NFK, spec.N, spec.K, k, b, 256, 32, part)
                                 for part in (qlr.PART_CODES, qlr.PART_C1_FP8, qlr.PART_S2))
        drawn.append(options.index((spec.bits, spec.block)))
        del W
    err[:] = out.cpu().numpy()
    budget = int(sum(cost[i, o] for i, o in enumerate(drawn)))
    t0 = time.perf_counter()
    choice, total = qlr.lqlora_allocate(err, cost, budget, 1 << 20)
    host_ms = 1e3 * (time.perf_counter() - t0)
    params = sum(s_.N * s_.K for s_ in wl.linears)
    hist = {}
    for o in choice:
        key = f"nf{options[o][0]}_b{options[o][1]}"
        hist[key] = hist.get(key, 0) + 1
    return {"options": [f"nf{k}_b{b}" for k, b in options], "error_pass_ms": gpu_ms, "allocate_ms": host_ms,
            "budget_bits_per_param": budget / params,
            "plan_bits_per_param": sum(cost[i, o] for i, o in enumerate(choice)) / params,
            "plan_total_sq_error": total, "seeded_draw_total_sq_error": float(sum(err[i, o] for i, o in enumerate(drawn))),
            "plan_histogram": hist, "unit_bits": 1 << 20}


# ------------------------------------------------------------------------------------------ decode shape
def run_decode(args, dev, steps, warmup):
    """Forward of the 28672 x 8192 NF4+DQ projection at 1, 4 and 16 tokens: HBM-bound on the codes.  Times
    the decode kernel alone (Y = X dequant(W)^T + T_save B^T) and the whole forward (T_save first)."""
    import numpy as np
    import torch
    from quantized_base_lora_nf4_b200 import qlr
    from synth import workload, linear_tensors

    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    wl = workload("decode70b", args.seed)
    spec = wl.linears[0]
    t = linear_tensors(spec, 16, seed=args.seed, with_dy=False)
    W = torch.from_numpy(t["W"]).to(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    quant = time_quantizer(qlr, spec, W, flush)
    quant["frac_of_hbm"] = quant["GBps"] / hbm
    q = qlr.quantize_nf4(W, 4, 64, 256)
    del W
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16).contiguous()  # noqa
    A, B = bf(t["A"]), bf(t["B"])
    code_bytes = spec.N * spec.K // 2
    all_bytes = code_bytes + spec.N * spec.K // 64 + 4 * spec.N * spec.K // (64 * 256) + 2 * spec.r * (spec.N + spec.K)
    out = {}
    for M in wl.token_counts:
        X = bf(t["X"][:M])
        ws = qlr.Workspace(dev)
        T = torch.empty((M, spec.r), dtype=torch.bfloat16, device=dev)
        Y = torch.empty((M, spec.N), dtype=torch.bfloat16, device=dev)
        for _ in range(warmup):
            qlr.lora_down(q, X, A, spec.s, T_save=T, ws=ws)
            qlr.forward_base(q, X, B, T, Y=Y)
        torch.cuda.synchronize()
        whole, kern = [], []
        for _ in range(steps):
            flush_l2(flush)
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
            qlr.lora_down(q, X, A, spec.s, T_save=T, ws=ws)
            e1.record()
            qlr.forward_base(q, X, B, T, Y=Y)
            e2.record()
            whole.append((e0, e2))
            kern.append((e1, e2))
        torch.cuda.synchronize()
        t_ms = statistics.median(a.elapsed_time(b) for a, b in whole)
        k_ms = statistics.median(a.elapsed_time(b) for a, b in kern)
        out[str(M)] = {"kernel_ms": k_ms, "kernel_code_GBps": code_bytes / k_ms / 1e6,
                       "kernel_code_frac_of_hbm": code_bytes / k_ms / 1e6 / hbm,
                       "kernel_all_GBps": all_bytes / k_ms / 1e6,
                       "forward_ms": t_ms, "forward_code_GBps": code_bytes / t_ms / 1e6,
                       "forward_code_frac_of_hbm": code_bytes / t_ms / 1e6 / hbm}
    return {"workload": "decode70b: NF4+DQ 28672x8192, r=64, forward at 1/4/16 tokens", "per_tokens": out,
            "target": "decode kernel at >= 0.70 of the HBM copy rate on the 4-bit code bytes (<= 25.7 us)",
            "quantizer": quant, "hbm_peak_gbs": hbm, "peak_kind": peak_kind,
            "code_bytes": code_bytes, "all_bytes": all_bytes,
            "timing": "median CUDA-event time over the timed repetitions, L2 flushed before each"}


def run_loqa(args, dev, peaks, peak_kind, steps, warmup):
    """LoQA's scale and zero-point gradients on the QA-LoRA layer (INT4 group 32, 4096 x 4096, 2048 tokens):
    a 2 M N K-flop contraction whose epilogue reduces each group with the codes."""
    import torch
    from quantized_base_lora_nf4_b200 import qlr
    from synth import workload, normal

    spec = workload("qalora").linears[0]
    M = workload("qalora").M
    W = torch.from_numpy(normal(args.seed, 0, "W", (spec.N, spec.K), spec.sigma_w, bf16=False)).to(dev)
    q = qlr.quantize_int4_group(W, spec.group)
    del W
    g = torch.Generator(device=dev)
    g.manual_seed(args.seed + 7)
    X = torch.randn((M, spec.K), generator=g, device=dev).to(torch.bfloat16)
    dY = torch.randn((M, spec.N), generator=g, device=dev).to(torch.bfloat16)
    dS = torch.empty((spec.N, spec.K // spec.group), dtype=torch.float32, device=dev)
    dZ = torch.empty_like(dS)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        qlr.loqa_grad(q, X, dY, dscale=dS, dzero=dZ)
    torch.cuda.synchronize()
    ev = []
    for _ in range(steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qlr.loqa_grad(q, X, dY, dscale=dS, dzero=dZ)
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    flops = 2.0 * M * spec.N * spec.K
    peak = float(peaks["bf16_tflops"])
    return {"workload": "loqa: dscale, dzero of the INT4 group-32 4096x4096 layer, 2048 tokens",
            "kernel": "loqa_grad_kernel", "ms": ms, "tflops": flops / (ms / 1e3) / 1e12,
            "frac_of_measured_burst": flops / (ms / 1e3) / 1e12 / peak, "peak_kind": f"{peak_kind} bf16 burst"}


# ------------------------------------------------------------------------------------------ main
def config_of(wl, world, seed):
    lin = [{"name": s.name, "N": s.N, "K": s.K, "r": s.r, "format": s.fmt, "bits": s.bits if s.fmt == "nfk" else 4,
            "block": s.block if s.fmt == "nfk" else s.group} for s in wl.linears]
    if len(lin) > 8:  # the stack: a summary
        hist = {}
        for d in lin:
            key = f"nf{d['bits']}_b{d['block']}"
            hist[key] = hist.get(key, 0) + 1
        lin = {"count": len(lin), "bits_block_histogram": hist}
    return {"workload": workload_desc(wl), "tokens_per_rank": wl.M, "linears": lin,
            "l2": "256 MiB buffer written, then read, before every timed step (L2 flushed, no dirty lines left); "
                  "the stack's activations (about 20 GB, every linear its own) are far larger than L2",
            "seed": seed, "parallelism": f"dp{world}"}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from synth import workload

    wl = workload("lqlora" if args.workload == "lqlora_init" else args.workload, args.seed)
    cfg = config_of(wl, world, args.seed)

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb = oracle_tokens_per_s(wl, args.seed)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wl.M / cb["value"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic", "config": cfg, "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if args.workload in ("lqlora_init", "decode70b"):
        if rank == 0:
            if args.workload == "lqlora_init":
                print(json.dumps(run_lqlora_init(args, dev)))
            else:
                print(json.dumps({"metric": "decode forward time and HBM GB/s on the 4-bit code bytes",
                                  **run_decode(args, dev, args.steps, args.warmup)}))
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    res = run_ours(args, args.workload, rank, world, dev, args.steps, args.warmup)
    quant = None
    if rank == 0:  # the quantiser path of the workload's first linear (memory-bound; HBM roofline)
        from quantized_base_lora_nf4_b200 import qlr
        spec0 = wl.linears[0]
        g = torch.Generator(device=dev)
        g.manual_seed(args.seed)
        Wq = torch.randn((spec0.N, spec0.K), generator=g, device=dev, dtype=torch.float32) * spec0.sigma_w
        quant = time_quantizer(qlr, spec0, Wq, torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev))
        del Wq
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_kind = load_peaks()
    s = summarize(res, world, peaks, peak_kind)
    line = {
        "metric": METRIC, "value": s.pop("value"), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": s.pop("ms_per_step"), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; the stack drawn on the device, the other workloads from numpy streams)",
        "config": cfg, **s,
        "quantizer": None if quant is None else {**quant, "bound": "hbm", "peak_GBps": float(peaks["hbm_gbs"]),
                                                 "frac": quant["GBps"] / float(peaks["hbm_gbs"])},
    }
    if world == 1 and not args.no_extra and args.workload == "lqlora":
        # the other configurations, each in its own timed run on the same GPU (not part of `value`)
        extra = {}
        for name, fused in (("qalora", False), ("mlp7b", False), ("mlp7b_swiglu_fused", True)):
            r = run_ours(args, name.split("_")[0], 0, 1, dev, steps=10, warmup=3, e2e_steps=5, swiglu_fused=fused)
            ss = summarize(r, 1, peaks, peak_kind)
            extra[name] = {"workload": workload_desc(r["wl"]), "tokens_per_s": ss["value"],
                           "ms_per_step": ss["ms_per_step"], "tflops": ss["tflops"],
                           "tc_frac_of_measured_burst": ss["tc_frac_of_measured_burst"],
                           "roofline": ss["roofline"], "step_breakdown_ms": ss["step_breakdown_ms"],
                           "e2e_tokens_per_s": ss["e2e"]["value"], "clocks": ss["clocks"],
                           "gpu_launches_per_step": ss["gpu_launches_per_step"]}
        extra["decode70b"] = run_decode(args, dev, steps=10, warmup=3)
        extra["loqa"] = run_loqa(args, dev, peaks, peak_kind, steps=10, warmup=3)
        line["extra"] = extra
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_tokens_per_s(wl, args.seed)
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
