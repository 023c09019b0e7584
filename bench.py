"""Benchmark of the QLoRA linear hot path on B200.

One step = forward + backward (Y, U, dX, dA, dB) of every linear of the
workload, on one batch of synthetic inputs already resident in HBM.  The
frozen weights are quantized once before timing (load time, as in training).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  Timing: CUDA events on the launching stream
around each step, L2 flushed (a 2x-L2 buffer write) between timed steps
outside the events, barrier + synchronize on both sides of the timed loop,
max over ranks.  Under torchrun each rank runs a data-parallel replica on
its own tokens and the adapter gradients dA/dB are summed across ranks with
NCCL every step (the one exchange data parallelism needs).

--impl reference times the CPU oracle (oracle/, plain C, fp64) on this
host's cores on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s (large R) & packed-weight HBM GB/s (small R), % roofline"
DEFAULT_WORKLOAD = "14b_layer"
OTHER_WORKLOADS = ["qwen3_0.6b_attn_qv", "8b_mlp"]


def algorithmic_flops(wl: synth.Workload, R: int) -> float:
    """4 R O I + 6 R r (I + O) per linear (fwd + bwd; no recompute, no decode ops)."""
    return float(sum(4.0 * R * l.O * l.I + 6.0 * R * wl.r * (l.I + l.O) for l in wl.linears))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------- clocks

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
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- GPU arm

class Layer:
    """Device buffers of one linear: quantized weight, adapters, inputs,
    outputs and workspaces (all allocated before timing).  dA and dB are
    views into the caller's flat gradient arena (one all-reduce per step)."""

    def __init__(self, q, torch, wl, li, R, rank_seed, dA, dB, host_outputs):
        lin = wl.linears[li]
        dev = "cuda"
        W = synth.weight(wl, li)
        A, B = synth.adapters(wl, li)
        Wd = torch.from_numpy(W).to(dev)
        self.w = q.qlora_quantize_nf4(Wd, wl.block, wl.group)
        del Wd
        self.A = torch.from_numpy(A).to(dev)
        self.B = torch.from_numpy(B).to(dev)
        # activations: per rank, distinct tokens (seeded), bf16
        xs = synth.normal(wl.seed(li, "X") + 7919 * rank_seed, (R, lin.I))
        ds = synth.normal(wl.seed(li, "dY") + 7919 * rank_seed, (R, lin.O))
        _, xb = synth.bf16_round(xs)
        _, db = synth.bf16_round(ds)
        del xs, ds
        xh = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
        dh = torch.from_numpy(db.view(np.int16)).view(torch.bfloat16)
        self.X = xh.to(dev)
        self.dY = dh.to(dev)
        self.x_host = xh.pin_memory() if host_outputs else None
        self.dy_host = dh.pin_memory() if host_outputs else None
        self.Y = torch.empty((R, lin.O), dtype=torch.bfloat16, device=dev)
        self.U = torch.empty((R, wl.r), dtype=torch.float32, device=dev)
        self.dX = torch.empty((R, lin.I), dtype=torch.bfloat16, device=dev)
        self.dA = dA
        self.dB = dB
        if host_outputs:  # the step's results, read back by the end-to-end pass
            self.y_host = torch.empty_like(self.Y, device="cpu").pin_memory()
            self.dx_host = torch.empty_like(self.dX, device="cpu").pin_memory()
        self.ws_f = q.workspace(q.qlora_linear_workspace_bytes(self.w, R, wl.r, 0, q.COMPUTE_BF16))
        self.ws_b = q.workspace(q.qlora_linear_workspace_bytes(self.w, R, wl.r, 1, q.COMPUTE_BF16))
        self.alpha = wl.alpha

    def step(self, q, X=None, dY=None):
        X = self.X if X is None else X
        dY = self.dY if dY is None else dY
        q.qlora_linear_fwd(self.w, X, self.A, self.B, self.alpha, Y=self.Y, U_out=self.U, ws=self.ws_f)
        q.qlora_linear_bwd(self.w, X, dY, self.A, self.B, self.alpha, U=self.U, dX=self.dX, dA=self.dA,
                           dB=self.dB, ws=self.ws_b)


class Model:
    """Every linear of a workload on this rank, with the adapter gradients
    of all of them in one flat fp32 arena."""

    def __init__(self, q, torch, wl, rank, host_outputs=False):
        R = wl.R
        sizes = [(wl.r * l.I, l.O * wl.r) for l in wl.linears]
        self.grads = torch.empty(sum(a + b for a, b in sizes), dtype=torch.float32, device="cuda")
        self.layers = []
        off = 0
        for li, (na, nb) in enumerate(sizes):
            lin = wl.linears[li]
            dA = self.grads[off:off + na].view(wl.r, lin.I)
            dB = self.grads[off + na:off + na + nb].view(lin.O, wl.r)
            off += na + nb
            self.layers.append(Layer(q, torch, wl, li, R, rank, dA, dB, host_outputs))
        if host_outputs:
            self.grads_host = torch.empty_like(self.grads, device="cpu").pin_memory()

    def step(self, q, dp, xs=None, dys=None):
        for i, L in enumerate(self.layers):
            L.step(q, None if xs is None else xs[i], None if dys is None else dys[i])
        dp.allreduce_flat(self.grads)


def measured_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    capture under profiles/, or None when there is none or the kernel's
    source has changed since it was taken (the capture records a hash of the
    source files)."""
    path = os.path.join(ROOT, "profiles", f"tc_qlinear_traffic_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for rel in rec.get("source_files", []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec.get("source_sha256"):
        return None
    k = rec.get("kernels", {}).get(kernel)
    return int(k["dram_bytes_per_launch"]) if k else None


def choose_peak(peaks, ms_per_step):
    """Roofline denominator: the measured burst bf16 figure for kernels in a
    short step, the sustained (seconds-long, power-capped) one when the
    kernels are timed inside a long step (>= 1 ms per step, repeated)."""
    if ms_per_step >= 1.0:
        return peaks["bf16_tflops_sustained"], f"{peaks['source']} bf16 dense (sustained: kernels timed inside a {ms_per_step:.1f} ms step)"
    return peaks["bf16_tflops"], f"{peaks['source']} bf16 dense (burst: kernels timed inside a {ms_per_step:.3f} ms step)"


def measure_step(q, torch, dist, dp, model, wl, world, steps, warmup, flush, peaks, sample_clocks=None):
    """Device-timed step of `model` (graph replays between CUDA events, L2
    flushed outside the events, max over ranks) plus the per-kernel pass.
    Returns the metrics of one workload."""
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(warmup):
        flush.zero_()
        model.step(q, dp)
    barrier()

    # One step is captured once in a CUDA graph (no host launch gaps in the
    # device timing) and replayed K times between CUDA events.  A second
    # graph of the same step, with the library's event pair around each
    # tensor-core GEMM launch, is then replayed K times for the per-kernel
    # durations; those events also hold each launch back until the one
    # before it has finished (no programmatic overlap), so the step time
    # comes from the first pass only.
    def capture():
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
            model.step(q, dp)
        torch.cuda.synchronize()
        return g

    n_before = q.qlora_kernel_launch_count()
    graph = capture()
    kernels_per_step = q.qlora_kernel_launch_count() - n_before
    for _ in range(warmup):
        flush.zero_()
        graph.replay()
    barrier()
    if sample_clocks is not None:
        sample_clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        graph.replay()
        ev[i][1].record(stream)
    barrier()
    clk = sample_clocks.stop() if sample_clocks is not None else None
    ms = dp.max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), device="cuda")
    del graph

    nrec = 16 * len(model.layers)
    q.qlora_kernel_timing_enable(nrec)
    tgraph = capture()
    tgraph.replay()  # warm-up; each replay re-records the same event pairs
    torch.cuda.synchronize()
    recs = []
    for i in range(steps):
        flush.zero_()
        tgraph.replay()
        torch.cuda.synchronize()
        try:
            recs.extend(q.qlora_kernel_timing_collect(nrec))
        except q.QLoraError as e:  # keep the step timing; report no roofline
            print(f"kernel timing unavailable: {e}", file=sys.stderr)
    del tgraph
    q.qlora_kernel_timing_enable(0)
    for L in model.layers:
        assert q.qlora_workspace_status(L.ws_f) == 0 and q.qlora_workspace_status(L.ws_b) == 0
    ms_per_step = ms / steps
    flops_step = algorithmic_flops(wl, wl.R)
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12

    by_kind = {}
    for kind, kms, kfl in recs:
        d = by_kind.setdefault(kind, [0.0, 0.0, 0])
        d[0] += kms
        d[1] += kfl
        d[2] += 1
    kernels = {}
    for kind, (kms, kfl, n) in sorted(by_kind.items()):
        name = "tc_qlinear_fwd" if kind == 0 else "tc_qlinear_dx"
        kernels[name] = {"launches": n, "ms_total": round(kms, 4),
                         "tflops": round(kfl / (kms * 1e-3) / 1e12, 2) if kms > 0 else None,
                         "share_of_step": round(kms / ms, 4) if ms > 0 else None}
    roofline = None
    if by_kind:
        kind, (kms, kfl, n) = max(by_kind.items(), key=lambda kv: kv[1][0])
        achieved = kfl / (kms * 1e-3) / 1e12
        peak, src = choose_peak(peaks, ms_per_step)
        kname = "tc_qlinear_fwd" if kind == 0 else "tc_qlinear_dx"
        roofline = {"bound": "tensor", "kernel": kname,
                    "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                    "frac": round(achieved / peak, 4), "traffic": measured_traffic(wl.name, kname),
                    "peak_source": src, "frac_of_burst_peak": round(achieved / peaks["bf16_tflops"], 4),
                    "flops_per_launch": kfl / n, "avg_launch_ms": kms / n}
    step_peak, step_src = choose_peak(peaks, ms_per_step)
    return {"ms_per_step": ms_per_step, "value": value, "kernels": kernels, "roofline": roofline,
            "kernels_per_step": int(kernels_per_step), "clocks": clk,
            "step_frac_of_peak": round(value / world / step_peak, 4),
            "step_frac_of_burst_peak": round(value / world / peaks["bf16_tflops"], 4),
            "step_peak_source": step_src}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import qlora_bit_frozen_b200 as q
    from qlora_bit_frozen_b200 import dp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    peaks = load_peaks()
    wl = synth.workload(args.workload, R=args.tokens if args.tokens > 0 else None)
    R = wl.R
    model = Model(q, torch, wl, rank, host_outputs=True)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    main = measure_step(q, torch, dist, dp, model, wl, world, args.steps, args.warmup, flush, peaks,
                        sample_clocks=clocks)
    launches = main["kernels_per_step"] * args.steps
    ms_per_step = main["ms_per_step"]
    flops_step = algorithmic_flops(wl, R)
    value = main["value"]

    # ---------------------------------------- end to end through the API
    # Every step copies its inputs X, dY in from pinned host memory and its
    # results back out: Y, dX of every linear and the summed adapter
    # gradients (the flat dA/dB arena).
    layers = model.layers
    h2d = sum(L.x_host.numel() * 2 + L.dy_host.numel() * 2 for L in layers)
    d2h = sum(L.Y.numel() * 2 + L.dX.numel() * 2 for L in layers) + model.grads.numel() * 4
    xs = [torch.empty_like(L.X) for L in layers]
    dys = [torch.empty_like(L.dY) for L in layers]

    def e2e_step():
        for L, X, dY in zip(layers, xs, dys):
            X.copy_(L.x_host, non_blocking=True)
            dY.copy_(L.dy_host, non_blocking=True)
        model.step(q, dp, xs, dys)
        for L in layers:
            L.y_host.copy_(L.Y, non_blocking=True)
            L.dx_host.copy_(L.dX, non_blocking=True)
        model.grads_host.copy_(model.grads, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(max(1, min(args.warmup, 3))):
        e2e_step()
    barrier()
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        flush.zero_()
        ee[i][0].record(stream)
        e2e_step()
        ee[i][1].record(stream)
    barrier()
    ems = dp.max_over_ranks(sum(a.elapsed_time(b) for a, b in ee), device="cuda")
    e2e_value = flops_step * world / (ems / e2e_steps * 1e-3) / 1e12
    del xs, dys, model
    torch.cuda.empty_cache()

    # --------------------------- the other large-R configurations, same rules
    others = {}
    for name in args.also:
        if name == wl.name:
            continue
        owl = synth.workload(name)
        om = Model(q, torch, owl, rank)
        r = measure_step(q, torch, dist, dp, om, owl, world, args.steps, args.warmup, flush, peaks)
        others[name] = {"value": round(r["value"], 3), "unit": "TFLOP/s", "ms_per_step": round(r["ms_per_step"], 5),
                        "tokens_per_gpu": owl.R, "r": owl.r,
                        "step_frac_of_peak": r["step_frac_of_peak"],
                        "step_frac_of_burst_peak": r["step_frac_of_burst_peak"],
                        "step_peak_source": r["step_peak_source"],
                        "roofline": r["roofline"], "kernels": r["kernels"],
                        "kernels_per_step": r["kernels_per_step"]}
        launches += r["kernels_per_step"] * args.steps
        del om
        torch.cuda.empty_cache()

    small = None
    if args.small_r and world == 1:
        small = run_small_r(q, torch, peaks, args)

    quant = None
    if world == 1:
        quant = time_quantize(q, torch, wl)

    export = None
    if world == 1 and args.export:
        try:
            export = time_export(q, torch, peaks)
        except (RuntimeError, ValueError) as e:  # reported in the line, not fatal to it
            export = {"error": str(e)[:300]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_rows if args.cpu_rows > 0 else default_sample_rows(wl))

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights and adapters)",
            "config": {"workload": wl.name, "tokens_per_gpu": R,
                       "linears": [[l.name, l.O, l.I] for l in wl.linears], "r": wl.r, "alpha": wl.alpha,
                       "nf4_block": wl.block, "dq_group": wl.group, "compute": "bf16, fp32 accumulate",
                       "parallelism": f"dp{world}" if world > 1 else "single GPU",
                       "l2": "flushed between timed steps (2x L2 write, outside the events)"},
            "step_frac_of_peak": main["step_frac_of_peak"],
            "step_frac_of_burst_peak": main["step_frac_of_burst_peak"],
            "step_peak_source": main["step_peak_source"],
            "roofline": main["roofline"], "kernels": main["kernels"],
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ems / e2e_steps, 5),
                    "steps": e2e_steps,
                    "copies": "X, dY in; Y, dX and the all-reduced dA/dB arena out, every step"},
            "clocks": main["clocks"], "gpu_launches": int(launches),
            "kernels_per_step": main["kernels_per_step"],
            "timing": "device step captured once in a CUDA graph and replayed; CUDA events around each replay; per-kernel durations from a second pass with events around each tensor-core launch",
            "other_configs": others,
            "small_r": small, "quantize": quant, "export": export,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_small_r(q, torch, peaks, args):
    """Bandwidth-bound regime: R in {1, 16, 128} against W [4096 x 4096] and
    [12288 x 4096], forward and dX, GB/s on packed weight bytes.  Formats:
    NF4 (B=64, C=256) and affine 4/8-bit with G in {32, 64, 128}.  Cold L2:
    rotating weight copies totalling >= 4x L2, captured in a CUDA graph.
    At 128 tokens the call is above the ridge point, so TFLOP/s (2 R O I
    per call) is reported beside GB/s."""
    out = {}
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size

    def clone(w):
        c = lambda t: None if t is None else t.clone()
        return q.QuantizedWeight(w.fmt, w.O, w.I, w.block, w.group, w.bits, c(w.codes),
                                 c(w.scale_codes), c(w.group_absmax), c(w.mean), c(w.scale),
                                 c(w.bias))

    for name in ("bw_sweep_4096", "bw_sweep_12288"):
        wl = synth.workload(name)
        lin = wl.linears[0]
        W = torch.from_numpy(synth.weight(wl, 0)).cuda()
        formats = [("", lambda: q.qlora_quantize_nf4(W, 64, 256))]
        for bits in (4, 8):
            for G in (32, 64, 128):
                formats.append((f"_affine{bits}_G{G}", lambda bits=bits, G=G: q.qlora_quantize_affine(W, bits, G)))
        A = torch.from_numpy(synth.adapters(wl, 0)[0]).cuda()
        B = torch.from_numpy(synth.adapters(wl, 0)[1]).cuda()
        for tag, make in formats:
            base = make()
            payload = base.payload_bytes()
            ncopy = max(2, math.ceil(4 * l2 / payload))
            copies = [base] + [clone(base) for _ in range(ncopy - 1)]
            for R in (1, 16, 128):
                X = torch.randn((R, lin.I), device="cuda").to(torch.bfloat16)
                dY = torch.randn((R, lin.O), device="cuda").to(torch.bfloat16)
                Y = torch.empty((R, lin.O), device="cuda", dtype=torch.bfloat16)
                dX = torch.empty((R, lin.I), device="cuda", dtype=torch.bfloat16)
                U = torch.empty((R, wl.r), device="cuda")
                wsf = q.workspace(q.qlora_linear_workspace_bytes(base, R, wl.r, 0, 1))
                wsb = q.workspace(q.qlora_linear_workspace_bytes(base, R, wl.r, 1, 1))
                res = {}
                for op in ("fwd", "dx"):
                    def call(w):
                        if op == "fwd":
                            q.qlora_linear_fwd(w, X, A, B, wl.alpha, Y=Y, U_out=U, ws=wsf)
                        else:
                            q.qlora_linear_bwd(w, None, dY, A, B, wl.alpha, U=U, want_da=False,
                                               want_db=False, dX=dX, ws=wsb)
                    for w in copies:
                        call(w)
                    torch.cuda.synchronize()
                    st = torch.cuda.Stream()
                    st.wait_stream(torch.cuda.current_stream())
                    g = torch.cuda.CUDAGraph()
                    reps = max(64, ncopy)
                    with torch.cuda.graph(g, stream=st):
                        for k in range(reps):
                            call(copies[k % ncopy])
                    torch.cuda.synchronize()
                    g.replay()
                    torch.cuda.synchronize()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    t_call = e0.elapsed_time(e1) / reps
                    gbs = payload / (t_call * 1e-3) / 1e9
                    # every other tensor the call touches, once: activations in
                    # and out (bf16), A and B (fp32), U written (fwd)
                    other = 2 * R * (lin.I + lin.O) + 4 * wl.r * (lin.I + lin.O)
                    if op == "fwd":
                        other += 4 * R * wl.r
                    tgbs = (payload + other) / (t_call * 1e-3) / 1e9
                    res[op] = {"us_per_call": round(t_call * 1e3, 3), "packed_GBps": round(gbs, 1),
                               "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                               "total_GBps": round(tgbs, 1),
                               "tflops": round(2.0 * R * lin.O * lin.I / (t_call * 1e-3) / 1e12, 3)}
                    del g
                out[f"{name}{tag}_R{R}"] = {"packed_bytes": int(payload), **res}
            del copies, base
            torch.cuda.empty_cache()
        del W
    out["peak_GBps"] = peaks["hbm_gbs"]
    out["peak_source"] = f"{peaks['source']} HBM copy bandwidth"
    out["timing"] = f"CUDA graph of >= 64 calls rotating weight copies >= 4x L2"
    return out


def time_quantize(q, torch, wl):
    """Load-time NF4 + double-quant encode of the workload's weights (ms)."""
    Ws = [torch.from_numpy(synth.weight(wl, li)).cuda() for li in range(len(wl.linears))]
    for W in Ws:
        q.qlora_quantize_nf4(W)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    qs = [q.qlora_quantize_nf4(W) for W in Ws]  # each synchronizes (reads the non-finite flag)
    dt = time.perf_counter() - t0
    n = sum(W.numel() for W in Ws)
    parts = {"codes": sum(w.codes.numel() for w in qs),
             "scale_codes": sum(w.scale_codes.numel() for w in qs),
             "group_absmax": sum(4 * w.group_absmax.numel() for w in qs),
             "mean": sum(4 * w.mean.numel() for w in qs)}
    total = sum(parts.values())
    return {"ms": round(dt * 1e3, 3), "weights": int(n), "GBps_fp32_in": round(n * 4 / dt / 1e9, 1),
            "payload_bytes": {**{k: int(v) for k, v in parts.items()}, "total": int(total),
                              "bits_per_weight": round(8 * total / n, 4)},
            "note": "host wall clock incl. the flag read-back synchronization"}


def time_export(q, torch, peaks):
    """The two lifecycle kernels around the layer, each timed with CUDA
    events around single launches, L2 flushed before each (outside the
    events): the fp32 export of an 8B-class MLP weight (12288 x 4096, r = 32)
    and one Adam step over the 1,146,880 adapter parameters of the Qwen3-0.6B
    q/v adapters."""
    O, I, r = 12288, 4096, 32
    w = q.qlora_quantize_nf4(torch.randn(O, I, device="cuda") * 0.02)
    A = torch.randn(r, I, device="cuda") * 0.02
    B = torch.randn(O, r, device="cuda") * 0.02
    out = torch.empty(O, I, device="cuda")
    n = 1146880
    p = torch.randn(n, device="cuda") * 0.02
    g = torch.randn(n, device="cuda") * 1e-2
    m = torch.zeros(n, device="cuda")
    v = torch.zeros(n, device="cuda")
    flush = torch.empty(2 * 126 * 2 ** 20 // 4, device="cuda")

    def timed(fn, reps):
        ms = []
        for i in range(reps):
            flush.fill_(float(i))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(i)
            e1.record()
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        ms.sort()
        return ms[len(ms) // 2]

    for i in range(3):
        q.qlora_merge(w, A, B, 2.0 * r, out=out)
        q.qlora_adam_step(p, g, m, v, i + 1, 1e-3)
    torch.cuda.synchronize()
    mms = timed(lambda i: q.qlora_merge(w, A, B, 2.0 * r, out=out), 10)
    ams = timed(lambda i: q.qlora_adam_step(p, g, m, v, i + 4, 1e-3), 20)
    mbytes = w.payload_bytes() + 4 * O * I + 4 * r * (O + I)
    abytes = 28 * n
    peak = peaks["hbm_gbs"]
    mg = mbytes / mms / 1e6
    ag = abytes / ams / 1e6
    return {
        "merge": {"shape": [O, I, r], "ms": round(mms, 4), "bytes": int(mbytes), "GBps": round(mg, 1),
                  "frac": round(mg / peak, 4)},
        "adam": {"params": n, "ms": round(ams, 4), "bytes": int(abytes), "GBps": round(ag, 1),
                 "frac": round(ag / peak, 4)},
        "peak_GBps": peak, "timing": "median of single launches, CUDA events, L2 flushed before each",
    }


# --------------------------------------------------------------- CPU oracle

def default_sample_rows(wl) -> int:
    """Tokens of the oracle's bounded sample: about 1e11 algorithmic flops
    (tens of seconds of fp64 work on a few host cores), 16..1024 tokens,
    never more than the workload has."""
    per_token = algorithmic_flops(wl, 1)
    rows = int(1e11 // per_token)
    rows = max(16, min(1024, rows))
    return min(rows, wl.R)


def cpu_baseline(wl, rows):
    """The oracle (plain C, fp64, OpenMP) on the first `rows` tokens of every
    linear: Y, U, dX, dA, dB.  TFLOP/s on the algorithmic flops of the sample."""
    import oracle
    R = min(rows, wl.R)
    t_total = 0.0
    for li in range(len(wl.linears)):
        W = synth.weight(wl, li)
        A, B = synth.adapters(wl, li)
        xw, _, dw, _ = synth.activations(wl, li, R)
        ow = oracle.quantize_nf4(W, wl.block, wl.group)
        t0 = time.perf_counter()
        oracle.linear_fwd(ow, xw, A, B, wl.r, wl.alpha)
        oracle.linear_bwd(ow, xw, dw, A, B, wl.r, wl.alpha)
        t_total += time.perf_counter() - t0
    fl = algorithmic_flops(wl, R)
    return {"value": round(fl / t_total / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(t_total, 3),
            "sample": f"first {R} of {wl.R} tokens of every linear of {wl.name}; Y, U, dX, dA, dB in fp64 "
                      f"(the rate is per algorithmic flop of the sample; the oracle's cost is linear in tokens)"}


def run_reference(args):
    """Reference arm: the CPU oracle, bounded row sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    wl = synth.workload(args.workload)
    R = min(args.ref_rows if args.ref_rows > 0 else default_sample_rows(wl), wl.R)
    prep = []
    for li in range(len(wl.linears)):
        W = synth.weight(wl, li)
        A, B = synth.adapters(wl, li)
        xw, _, dw, _ = synth.activations(wl, li, R)
        prep.append((oracle.quantize_nf4(W, wl.block, wl.group), xw, dw, A, B))

    def step():
        for ow, xw, dw, A, B in prep:
            oracle.linear_fwd(ow, xw, A, B, wl.r, wl.alpha)
            oracle.linear_bwd(ow, xw, dw, A, B, wl.r, wl.alpha)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    fl = algorithmic_flops(wl, R)
    value = fl * args.steps / dt / 1e12
    sample = f"first {R} of {wl.R} tokens of every linear of {wl.name} per step; Y, U, dX, dA, dB in fp64"
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "tokens_sampled": R, "r": wl.r, "alpha": wl.alpha},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def launch_ranks(args, argv):
    """--gpus N > 1 outside a torchrun launch: start N ranks on this node
    (one per GPU) with torch.distributed.run on 127.0.0.1 and return its
    exit status."""
    import socket
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd, cwd=ROOT)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.WORKLOADS[1:])
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count per GPU (0: the workload's own)")
    ap.add_argument("--also", nargs="*", default=None,
                    help="other large-R workloads timed the same way into other_configs "
                         "(default: the Qwen3-0.6B q/v and 8B MLP configurations)")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="tokens of the CPU-baseline sample (0: a bounded sample of about 1e11 flops)")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="tokens per step of the reference arm (0: the same bounded sample size)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-r", dest="small_r", action="store_false")
    ap.add_argument("--no-export", dest="export", action="store_false",
                    help="skip timing the fp32 export (merge) and the adapter Adam step")
    ap.add_argument("--print-ranks", action="store_true",
                    help="each rank prints its RANK/WORLD_SIZE as JSON and exits (checks the launcher)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.also is None:
        args.also = list(OTHER_WORKLOADS)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args, argv))
    if args.print_ranks:
        print(json.dumps({"rank": int(os.environ.get("RANK", "0")),
                          "world": int(os.environ.get("WORLD_SIZE", "1")),
                          "local_rank": int(os.environ.get("LOCAL_RANK", "0"))}), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
