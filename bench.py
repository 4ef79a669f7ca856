#!/usr/bin/env python
"""Benchmark of the fused HEA forward + adjoint-gradient path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload hea_20q_L100]

One step = one training step on one synthetic batch: the fused forward pass
(encoding, every layer, checkpoint slots, <Z0>), the loss seed, and the fused
adjoint backward pass (every gradient).  Inputs are resident in HBM before the
timed region; the 512 MiB working state of the default workload is larger than
L2, so no flush is needed between steps.  For N > 1 every rank runs its own
batch (weak scaling) and the gradients are summed with one NCCL all-reduce per
step, as data-parallel training does.

--impl reference times the CPU oracle (complex128, gate by gate) on the host
cores instead: there is no other runnable implementation of this method.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from adjoint_gradients_b200.inputs import WORKLOADS, draw_theta, draw_x, draw_y  # noqa: E402

METRIC = "HEA samples/sec (fwd + adjoint grad), 20q; achieved HBM GB/s vs B200 peak"
UNIT = "samples/s"
# FP32 ALU roofline: 148 SMs x 128 FP32 lanes x 2 flop (FMA) x 1965 MHz max SM clock.
SMS, FP32_LANES, SM_MAX_MHZ = 148, 128, 1965.0
ALU_PEAK_TFLOPS = SMS * FP32_LANES * 2 * SM_MAX_MHZ * 1e6 / 1e12
HBM_NOMINAL_GBS = 8000.0  # B200 data-sheet HBM3e bandwidth (context; the roofline uses the measured copy)
FP64_LANES = 64       # FP64 FMA lanes per SM (B200 data sheet: 40 TFLOP/s FP64 at boost)
ALU64_PEAK_TFLOPS = SMS * FP64_LANES * 2 * SM_MAX_MHZ * 1e6 / 1e12
FMA_FWD_PER_ROT = 8   # per amplitude: one fused SU(2) on a pair = 16 FMA / 2 amplitudes
FMA_BWD_PER_ROT = 22  # per amplitude: U^dagger on psi (8) and lambda (8) + three Im<l|P|p> terms (6)
# split form (qml_split_form): per amplitude and rotation, Ry in tangent form
# on a pair = 4 FMA / 2 amplitudes; backward the same on psi and lambda (4)
# plus the three Im<l|P|p> terms (6).  Per amplitude and diagonal op: the
# complex factor (4 FMA, shared by the two lanes of a pair) and its product
# with each lane (4 FMA per complex value): forward 2 + 4, backward 4 + 8.
FMA_FWD_PER_RY, FMA_BWD_PER_RY = 2, 10
FMA_FWD_PER_DIAG, FMA_BWD_PER_DIAG = 6, 12
CPU_SAMPLE_LAYERS = 16  # oracle sample depth (cost is linear in depth)


def kernel_sources_digest():
    """sha256 over the sources of the pass kernels (ties recorded counters to a build)."""
    import hashlib

    h = hashlib.sha256()
    for rel in ("pass_kernel.cuh", "pass_split.cu", "kernels.cu", "device_plan.h", "plan.cpp"):
        with open(os.path.join(ROOT, "adjoint_gradients_b200", "csrc", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                "clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- helpers

def algorithmic_counts(ctx, w, B, f64=False, cnot_passes_per_layer=0):
    """Algorithmic FMAs and HBM bytes per step of the forward and backward pass kernels."""
    sched = ctx.debug_schedule()
    P = sched[0]
    N = 1 << w.n
    amp = B * N
    rots = w.n * w.L
    if ctx.split_form and ctx.cnot_fused:  # fused CNOT schedule: two diagonal ops per layer and qubit set
        fma_f = FMA_FWD_PER_RY * rots + FMA_FWD_PER_DIAG * 4 * w.L
        fma_b = FMA_BWD_PER_RY * rots + FMA_BWD_PER_DIAG * 4 * w.L
    elif ctx.split_form:  # one diagonal op per layer boundary (forward: also the one before layer 0)
        # fp64 mode keeps one sample per tile: its forward factor is not shared by two lanes (4 + 4)
        fma_f = FMA_FWD_PER_RY * rots + (8 if f64 else FMA_FWD_PER_DIAG) * (w.L + 1)
        fma_b = FMA_BWD_PER_RY * rots + FMA_BWD_PER_DIAG * w.L
    else:
        fma_f, fma_b = FMA_FWD_PER_ROT * rots, FMA_BWD_PER_ROT * rots
    if cnot_passes_per_layer:  # CNOT entanglers: every layer's passes read and write the state once
        Pc = cnot_passes_per_layer * w.L
        c = 16 if f64 else 8
        return {"passes": Pc, "fwd_fma": fma_f * amp, "bwd_fma": fma_b * amp,
                "fwd_bytes": (2 * c * Pc - c) * amp, "bwd_bytes": (4 * c * Pc - 2 * c) * amp}
    # bytes per amplitude moved by each pass, from the schedule flags
    i = 1
    fwd_bytes = bwd_bytes = 0
    slot_b = {"bf16": 4, "fp32": 8, "fp64": 16}[w.storage]
    c = 16 if f64 else 8  # one complex amplitude
    for _ in range(P):
        set_id, gen, last, ck, nops = sched[i:i + 5]
        i += 5 + 4 * nops
        fwd_bytes += (0 if gen else c) + c + (slot_b if ck >= 0 else 0)
        if f64:  # psi and lambda read (the slot replaces psi at a boundary) and written
            bwd_bytes += 2 * c + (slot_b - c if ck >= 0 else 0) + (0 if gen else 2 * c)
            continue
        rd = 8 if last else 16
        wr = 0 if gen else 16
        bwd_bytes += rd + wr + (slot_b if ck >= 0 else 0)
    return {
        "passes": P,
        "fwd_fma": fma_f * amp,
        "bwd_fma": fma_b * amp,
        "split": bool(ctx.split_form),
        "fwd_bytes": fwd_bytes * amp,
        "bwd_bytes": bwd_bytes * amp,
    }


def oracle_sample(w, layers, rank=0):
    """Time the oracle (forward + adjoint) on one sample of the workload at reduced depth."""
    import oracle

    x = draw_x(w.index, 1, w.n)
    theta = draw_theta(w.index, w.L, w.n)[:layers]
    y = draw_y(w.index, 1)
    t0 = time.perf_counter()
    E = oracle.forward(x, theta)
    oracle.adjoint(x, theta, oracle.loss_seed(E, y))
    return time.perf_counter() - t0, oracle.num_threads()


def cpu_baseline(w):
    t, cores = oracle_sample(w, CPU_SAMPLE_LAYERS)
    per_sample = t * w.L / CPU_SAMPLE_LAYERS
    return {
        "value": 1.0 / per_sample, "unit": UNIT, "cores": cores, "kind": "oracle",
        "sample": (f"1 sample of {w.name} at {CPU_SAMPLE_LAYERS} of {w.L} layers "
                   f"({t:.1f} s), scaled x{w.L / CPU_SAMPLE_LAYERS:g} to full depth"),
    }


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def physical_gpu(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[local])
        except (ValueError, IndexError):
            return local
    return local


# ---------------------------------------------------------------------------- arms

def run_reference(args):
    world, rank, _ = dist_env()
    w = WORKLOADS[args.workload]
    if rank != 0:
        return 0
    layers = max(1, min(w.L, args.ref_layers))
    for _ in range(args.warmup):
        oracle_sample(w, layers)
    times = []
    cores = 1
    for _ in range(args.steps):
        t, cores = oracle_sample(w, layers)
        times.append(t)
    per_step = float(np.mean(times))
    per_sample = per_step * w.L / layers
    value = 1.0 / per_sample
    sample = f"1 sample of {w.name} at {layers} of {w.L} layers per step, scaled x{w.L / layers:g} to full depth"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**workload_config(w, w.B), "parallelism": "single", "observable": "Z0",
                   "entangler": f"CZ chain ({w.n - 1} bonds)", "reupload": False},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, B, f64=False):
    return {
        "workload": w.name, "n_qubits": w.n, "layers": w.L, "batch_per_gpu": B, "params": w.params,
        "ckpt_block": w.ckpt_block, "ckpt_storage": w.storage,
        "state": "complex128 [B][2^n]" if f64 else "complex64 [B][2^n]",
        "l2": (f"inputs larger than L2 (working state B*2^n*{16 if f64 else 8} B > 126 MB); no flush"),
        "seeds": {"x": 1000 + w.index, "theta": 2000 + w.index, "y": 3000 + w.index},
    }


def observable_terms(name, n):
    """[(coef, word)] for --observable (letter q acts on qubit q), or None for Z0."""
    if name == "z0":
        return None
    out = []
    for q in range(n - 1):
        w = ["I"] * n
        w[q] = w[q + 1] = "Z"
        out.append((1.0, "".join(w)))
    for q in range(n):
        w = ["I"] * n
        w[q] = "X"
        out.append((0.9, "".join(w)))
    return out


def entangler_bonds(name, n):
    """Pairs for --entangler (CZ bonds, or (control, target) for the CNOT ladder)."""
    chain = [(q, q + 1) for q in range(n - 1)]
    return {"chain": chain, "ring": chain + [(n - 1, 0)], "none": [], "cnot": chain}[name]


def entangler_kind(name):
    return "cnot" if name == "cnot" else "cz"


def run_ours(args):
    import torch

    from adjoint_gradients_b200 import qml

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import dataclasses

    w = WORKLOADS[args.workload]
    f64 = args.precision == "fp64"
    if f64:  # fp64 mode keeps its checkpoint slots exact
        w = dataclasses.replace(w, storage="fp64")
    if args.ckpt_block is not None:  # checkpoint-block sweeps
        w = dataclasses.replace(w, ckpt_block=args.ckpt_block)
    fdt = torch.float64 if f64 else torch.float32
    B = w.B
    dev = f"cuda:{local}"
    # each rank draws its own batch; theta is shared
    x = np.random.default_rng(1000 + w.index + 7919 * rank).uniform(0, np.pi, (B, w.n))
    y = np.random.default_rng(3000 + w.index + 7919 * rank).integers(0, 2, B) * 2.0 - 1.0
    theta = draw_theta(w.index, w.L, w.n)
    xd = torch.tensor(x, dtype=fdt, device=dev)
    yd = torch.tensor(y, dtype=fdt, device=dev)
    td = torch.tensor(theta, dtype=fdt, device=dev)

    ctx = qml.Context(w.n, w.L, B, ckpt_block=w.ckpt_block, storage=w.storage, device=local,
                      precision=args.precision)
    obs = observable_terms(args.observable, w.n)
    ctx.set_observable(obs)
    bonds = entangler_bonds(args.entangler, w.n)
    ctx.set_entangler(bonds, kind=entangler_kind(args.entangler))
    ctx.set_reupload(args.reupload)
    psi = ctx.new_state(B)
    lam = ctx.new_state(B)
    E = torch.empty(B, dtype=fdt, device=dev)
    grad = torch.empty((w.L, w.n, 3), dtype=fdt, device=dev)
    stream = torch.cuda.current_stream()

    from adjoint_gradients_b200 import dp

    def step():
        ctx.forward(td, xd, psi, E)
        g, _ = ctx.loss_seed(E, yd)
        ctx.backward(td, xd, psi, lam, g, grad)
        if dist is not None:
            dp.average_gradients(grad)

    for _ in range(args.warmup):
        step()
    ctx.sync()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    # One GPU: the step (forward, loss seed, backward) is captured once into a
    # CUDA graph and the timed region replays it, so small circuits are not
    # bound by the host's per-launch cost.  The pass kernels' event spans are
    # captured with it and read after the replays (the last step's).
    graph = None
    timed_steps_in_spans = args.steps
    ctx.enable_timing(True)
    if world == 1 and not args.no_graph:
        step()  # an eager timed step: the span events exist before the capture
        torch.cuda.synchronize()
        ctx.read_timing()
        try:
            l0 = ctx.launch_count
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                step()
            graph, per_step = g, ctx.launch_count - l0
            g.replay()
            torch.cuda.synchronize()
            timed_steps_in_spans = 1
        except Exception as exc:  # noqa: BLE001 - reported; the eager loop is timed instead
            print(f"graph capture failed, timing the eager loop: {exc}", file=sys.stderr)
            graph = None
            torch.cuda.synchronize()
    if graph is None:
        ctx.read_timing()  # start the eager loop's spans empty (a graph keeps its captured ones)
    clocks = ClockSampler(physical_gpu(local))
    clocks.start()
    time.sleep(0.3)
    launches0 = ctx.launch_count
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    launches = (per_step * args.steps) if graph is not None else ctx.launch_count - launches0
    try:
        fwd_ms, fwd_n, bwd_ms, bwd_n = ctx.read_timing()
    except qml.QmlError as exc:  # spans inside the graph unreadable: take them from an eager loop
        if graph is None:
            raise
        print(f"graph spans unreadable ({exc}); pass-kernel spans from an eager loop", file=sys.stderr)
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        fwd_ms, fwd_n, bwd_ms, bwd_n = ctx.read_timing()
        timed_steps_in_spans = args.steps
    ctx.enable_timing(False)
    clk = clocks.stop()
    ctx.sync()
    ms = ev0.elapsed_time(ev1)
    if dist is not None:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    value = world * B * args.steps / (ms / 1e3)

    # ---- ALU peaks measured on this GPU (independent FMA chains over every SM;
    # qml_measure_fma_peak), beside the ones derived from unit counts
    meas = {}
    for name, is64 in (("fp32x2", False), ("fp64", True)):
        try:
            meas[name] = qml.measure_fma_peak(is64, 100000)[0]
        except Exception as exc:  # noqa: BLE001 - reported, not fatal
            meas[name] = None
            print(f"fma peak measurement failed: {exc}", file=sys.stderr)

    # ---- roofline of the dominant kernel (the backward pass kernel)
    cnot_ppl = 0
    if args.entangler == "cnot" and not ctx.cnot_fused:  # passes per layer of the one-layer schedule = the set count
        cnot_ppl = (w.n + 9) // 10 if w.n > 12 else 1
    cnt = algorithmic_counts(ctx, w, B, f64, cnot_ppl)
    hbm_peak, peak_src = measured_peaks()
    # fp32: the peak derived from unit counts and the clock; fp64: the
    # measured DFMA peak (the unit count of the FP64 pipe is not published
    # for this part), derived value beside it
    alu_peak = (meas["fp64"] or ALU64_PEAK_TFLOPS) if f64 else ALU_PEAK_TFLOPS
    bwd_avg_s = bwd_ms / 1e3 / max(1, bwd_n)
    fwd_avg_s = fwd_ms / 1e3 / max(1, fwd_n)
    # per step: the pass kernels' algorithmic work over their summed event time
    bwd_step_s = bwd_ms / 1e3 / timed_steps_in_spans
    fwd_step_s = fwd_ms / 1e3 / timed_steps_in_spans
    bwd_tflops = 2 * cnt["bwd_fma"] / bwd_step_s / 1e12
    fwd_tflops = 2 * cnt["fwd_fma"] / fwd_step_s / 1e12
    bwd_gbs = cnt["bwd_bytes"] / bwd_step_s / 1e9
    fwd_gbs = cnt["fwd_bytes"] / fwd_step_s / 1e9
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        with open(tfile) as f:
            tr = json.load(f).get(w.name, {})
        # counters taken on another build of the kernels do not count
        default_path = not f64 and args.entangler == "chain" and not args.reupload and obs is None
        if tr.get("kernel_sources_sha256") == kernel_sources_digest() and default_path:
            traffic = tr.get("bwd_pass_bytes_per_launch")
    # the bound is the resource the dominant kernel uses the larger fraction of
    hbm_bound = bwd_gbs / hbm_peak > bwd_tflops / alu_peak
    roofline = {
        "kernel": "pass64_kernel<backward>" if f64 else "pass_kernel<backward>",
        "bound": "hbm" if hbm_bound else "alu",
        "achieved": bwd_gbs if hbm_bound else bwd_tflops, "peak": hbm_peak if hbm_bound else alu_peak,
        "unit": "GB/s" if hbm_bound else "TFLOP/s",
        "frac": bwd_gbs / hbm_peak if hbm_bound else bwd_tflops / alu_peak, "traffic": traffic,
        "alu_achieved_tflops": bwd_tflops, "alu_peak_tflops": alu_peak, "alu_frac": bwd_tflops / alu_peak,
        "fma_per_step": cnt["bwd_fma"], "bytes_per_step": cnt["bwd_bytes"], "split_form": cnt.get("split", False),
        "peak_src": (("measured: independent DFMA chains on every SM (qml_measure_fma_peak); derived "
                      f"148 SMs x 64 FP64 lanes x 2 x 1965 MHz = {ALU64_PEAK_TFLOPS:.2f}") if f64 and meas["fp64"] else
                     "148 SMs x 64 FP64 lanes x 2 x 1965 MHz (DFMA; derived from unit counts)" if f64 else
                     "148 SMs x 128 FP32 lanes x 2 x 1965 MHz (FFMA; packed f32x2 FMA measured at the same rate)"),
        "alu_peak_measured_tflops": meas,
        "avg_launch_ms": bwd_avg_s * 1e3, "launches": bwd_n,
        "hbm_achieved_gbs": bwd_gbs, "hbm_peak_gbs": hbm_peak, "hbm_frac": bwd_gbs / hbm_peak,
        "hbm_frac_of_nominal_8000": bwd_gbs / HBM_NOMINAL_GBS,
        "hbm_peak_src": peak_src,
        "forward_kernel": {"achieved_tflops": fwd_tflops, "frac": fwd_tflops / alu_peak,
                           "hbm_gbs": fwd_gbs, "hbm_frac": fwd_gbs / hbm_peak,
                           "hbm_frac_of_nominal_8000": fwd_gbs / HBM_NOMINAL_GBS, "avg_launch_ms": fwd_avg_s * 1e3},
    }

    # ---- end to end through host buffers (pinned), same metric
    e2e = None
    if not args.no_e2e:
        ctx_h = qml.Context(w.n, w.L, B, ckpt_block=w.ckpt_block, storage=w.storage, device=local, host_step=True,
                            precision=args.precision)
        ctx_h.set_observable(obs)
        ctx_h.set_entangler(bonds, kind=entangler_kind(args.entangler))
        ctx_h.set_reupload(args.reupload)
        xh = torch.tensor(x, dtype=fdt).pin_memory()
        th = torch.tensor(theta, dtype=fdt).pin_memory()
        yh = torch.tensor(y, dtype=fdt).pin_memory()
        out = qml.StepResult(torch.empty(B, dtype=fdt).pin_memory(), torch.empty(1, dtype=fdt).pin_memory(),
                             torch.empty((w.L, w.n, 3), dtype=fdt).pin_memory())
        for _ in range(max(1, min(args.warmup, 2))):
            ctx_h.step_host(xh, th, yh, out)
        k2 = max(1, args.steps)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k2):
            ctx_h.step_host(xh, th, yh, out)
            if dist is not None:
                gt = out.grad.to(dev, non_blocking=False)
                dp.average_gradients(gt)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        if dist is not None:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        fb = 8 if f64 else 4
        h2d = fb * (B * w.n + w.L * w.n * 3 + B)
        d2h = fb * (B + 1 + w.L * w.n * 3)
        e2e = {"value": world * B * k2 / (ems / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "api": "qml_step_host"}
        ctx_h.sync()
        del ctx_h

    # ---- one real epoch: samples_per_epoch samples in mini-batches of B, the
    # short last batch run as it is (its own x and y), timed on the device
    epoch = None
    if args.epoch and w.samples_per_epoch:
        S = w.samples_per_epoch
        xe = np.random.default_rng(1000 + w.index + 7919 * rank).uniform(0, np.pi, (S, w.n))
        ye = np.random.default_rng(3000 + w.index + 7919 * rank).integers(0, 2, S) * 2.0 - 1.0
        batches = [(i, min(B, S - i)) for i in range(0, S, B)]
        xb = [torch.tensor(xe[i:i + b], dtype=fdt, device=dev) for i, b in batches]
        yb = [torch.tensor(ye[i:i + b], dtype=fdt, device=dev) for i, b in batches]
        torch.cuda.reset_peak_memory_stats(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        for (i, b), xi, yi in zip(batches, xb, yb):
            Ei = E[:b]
            ctx.forward(td, xi, psi[:b], Ei)
            gi, _ = ctx.loss_seed(Ei, yi)
            ctx.backward(td, xi, psi[:b], lam[:b], gi, grad)
            if dist is not None:
                dp.average_gradients(grad)
        q1.record(stream)
        torch.cuda.synchronize()
        ctx.sync()
        es = q0.elapsed_time(q1) / 1e3
        if dist is not None:
            t = torch.tensor([es], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            es = float(t.item())
        epoch = {"s_per_epoch_measured": es, "samples": S, "batches": [b for _, b in batches][-2:],
                 "n_batches": len(batches), "peak_hbm_bytes_epoch": int(torch.cuda.max_memory_allocated(dev))}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    cfg = {**workload_config(w, B, f64), "parallelism": f"dp{world}" if world > 1 else "single",
           "observable": "Z0" if obs is None else f"{args.observable} ({len(obs)} Pauli strings)",
           "entangler": (f"CNOT ladder ({len(bonds)} pairs, "
                         f"{'fused into the rotation passes' if ctx.cnot_fused else 'one gather pass per layer'})"
                         if args.entangler == "cnot" else
                         f"CZ {args.entangler} ({len(bonds)} bonds)"),
           "reupload": bool(args.reupload)}
    # how this arm ran (kept out of config, which both arms report alike)
    run = {"cuda_graph": graph is not None, "peak_hbm_bytes": int(torch.cuda.max_memory_allocated(dev))}
    if w.samples_per_epoch:
        run["s_per_epoch"] = w.samples_per_epoch / (value / world)
        run["epoch"] = f"{w.samples_per_epoch} samples per GPU at the measured samples/s (mini-batch {B})"
    if epoch is not None:
        run["epoch_run"] = epoch
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64" if f64 else "f32", "data": "synthetic",
            "config": cfg, "run": run,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="hea_20q_L100", choices=sorted(WORKLOADS) + ["custom"])
    ap.add_argument("--ref-layers", type=int, default=2)
    ap.add_argument("--case", default=None,
                    help="n,L,B[,ckpt_block[,storage]]: a custom shape with the workload's seeds (for profiling)")
    ap.add_argument("--observable", default="z0", choices=["z0", "tfim"],
                    help="z0: <Z0> (the workloads' readout); tfim: sum_q Z_q Z_q+1 + 0.9 sum_q X_q")
    ap.add_argument("--entangler", default="chain", choices=["chain", "ring", "none", "cnot"],
                    help="gates ending every layer: CZ chain (q, q+1) as in the workloads, CZ ring, none, "
                         "or the CNOT ladder (q -> q+1)")
    ap.add_argument("--reupload", action="store_true", help="data re-uploading: the encoding again in every layer")
    ap.add_argument("--precision", default="fp32", choices=["fp32", "fp64"],
                    help="arithmetic of the path: fp32, or fp64 (complex128 state, exact checkpoint slots)")
    ap.add_argument("--ckpt-block", type=int, default=None,
                    help="override the workload's checkpoint block (layers per block; 0: none)")
    ap.add_argument("--epoch", action="store_true",
                    help="also time one real epoch of the workload (its samples in mini-batches, short last batch as is)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time the eager launch loop instead of a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.case:
        from adjoint_gradients_b200.inputs import Workload

        f = args.case.split(",")
        n, L, B = int(f[0]), int(f[1]), int(f[2])
        ck = int(f[3]) if len(f) > 3 else 0
        st = f[4] if len(f) > 4 else "fp32"
        WORKLOADS["custom"] = Workload(WORKLOADS[args.workload].index, f"custom_{n}q_L{L}_B{B}", n, L, B, ck, st)
        args.workload = "custom"
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
