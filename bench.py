#!/usr/bin/env python
"""Benchmark of the KronQ per-sublayer quantization engine on B200.

One step = one full sublayer quantization through libkronq's C ABI:
covariance of the calibration activations X and of the output gradients G,
sensitivity, BiIP, damped inverse Cholesky factor, blocked OBS with packing.
Default workload: a LLaMA-3-70B down_proj-shaped sublayer (W 8192 x 28672,
131072 calibration tokens, W2 g128, synthetic seeded inputs).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Multi-GPU runs quantize one independent
sublayer per rank (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("sublayer quantize time (ms) & TFLOP/s: cov accum + BiIP + Cholesky "
          "+ blocked OBS")
DEFAULT_WORKLOAD = "llama3_70b_down_8192x28672"


def algorithmic_flops(wl):
    """Per-sublayer work the method must do: covariances n*d*(d+1) (one
    triangle), Cholesky + inverse 2d^3/3, OBS updates d_out*d_in*(d_in-1)."""
    n, di, do = wl.n, wl.d_in, wl.d_out
    parts = {"cov_x": n * di * (di + 1), "cov_g": n * do * (do + 1),
             "chol": 2 * di ** 3 / 3, "quant": do * di * (di - 1)}
    return parts, float(sum(parts.values()))


def biip_bytes(wl):
    """Two read+write passes per rotated matrix (H_X, H_G in fp32; W read in
    bf16 and written in fp32, then one more fp32 pass)."""
    return 16 * wl.d_in ** 2 + 16 * wl.d_out ** 2 + 14 * wl.d_out * wl.d_in


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def load_traffic(kernel, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if present."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    try:
        with open(path) as f:
            return json.load(f).get("dram_bytes_per_launch")
    except OSError:
        return None


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200", "-i", self.uuid],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- oracle sample
def oracle_sample(wl):
    """Times the fp64 oracle, as it stands, on a bounded sample of the
    workload and extrapolates each step to full size by its cost model.
    Returns (seconds for one full sublayer, description, threads)."""
    import numpy as np
    import torch

    import oracle as O
    from second_order_post_b200 import synth

    t = {}
    ns = min(wl.n, 131072)
    for key, d, rng in (("cov_x", wl.d_in, wl.x_range), ("cov_g", wl.d_out, wl.g_range)):
        a = synth.make_activations(ns, 256, *rng, wl.dtype, seed=11).float().numpy()
        t0 = time.perf_counter()
        O.cov(a)
        dt = time.perf_counter() - t0
        t[key] = dt * (wl.n * d * (d + 1)) / (ns * 256 * 257)
    # BiIP: dense rotations, cubic in the dimensions; sample at 1/16 size
    fo = 16 if wl.d_out >= 2048 else 1
    fi = 16 if wl.d_in >= 2048 else 1
    do_s, di_s = wl.d_out // fo, wl.d_in // fi
    rin = (wl.rot_in[0] // fi, wl.rot_in[1]) if wl.rot_in[0] % fi == 0 else (di_s, 1)
    rout = (wl.rot_out[0] // fo, wl.rot_out[1]) if wl.rot_out[0] % fo == 0 else (do_s, 1)
    w = np.random.default_rng(1).standard_normal((do_s, di_s)) * 0.02
    hx = synth.make_spd(di_s, seed=1).double().numpy()
    hg = synth.make_spd(do_s, seed=2).double().numpy()
    t0 = time.perf_counter()
    O.biip(w, hx, hg, seed=0, rot_in=rin, rot_out=rout)
    dt = time.perf_counter() - t0
    cost = lambda a, b: a * a * b + a * b * b + 2 * a ** 3 + 2 * b ** 3
    t["biip"] = dt * cost(wl.d_out, wl.d_in) / cost(do_s, di_s)
    ds = min(2048, wl.d_in)
    h = synth.make_spd(ds, seed=3).double().numpy()
    t0 = time.perf_counter()
    O.chol_inv(h, 0.01)
    t["chol"] = (time.perf_counter() - t0) * (wl.d_in / ds) ** 3
    rows, dq = min(256, wl.d_out), min(2048, wl.d_in)
    u = np.triu(np.random.default_rng(2).standard_normal((dq, dq)) * 0.01)
    np.fill_diagonal(u, 1.0)
    ws = np.random.default_rng(3).standard_normal((rows, dq)) * 0.02
    t0 = time.perf_counter()
    O.obs_quantize(ws, u, wl.bits, wl.group)
    t["quant"] = (time.perf_counter() - t0) * (wl.d_out / rows) * (wl.d_in / dq) ** 2
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        nt = [i.get("num_threads", 0) for i in threadpool_info()
              if i.get("user_api") == "blas"]
        if nt:
            threads = max(nt)
    except Exception:
        pass
    desc = (f"cov: one 256x256 block of H over {ns} tokens per side; BiIP: "
            f"{do_s}x{di_s} sublayer; Cholesky: {ds}^2; OBS: {rows} rows x "
            f"{dq} columns; each extrapolated to full size by its flop count "
            f"(cubic for the dense BiIP/Cholesky, rows*d^2 for OBS)")
    del torch
    return sum(t.values()), desc, threads, t


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    _, flops = algorithmic_flops(wl)
    for _ in range(args.warmup):
        oracle_sample(wl)
    secs = []
    for _ in range(args.steps):
        s, desc, threads, _ = oracle_sample(wl)
        secs.append(s)
    sec = statistics.mean(secs)
    value = flops / sec / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": workload_config(wl, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": desc, "cpu_model": cpu_model(),
                         "nproc": os.cpu_count()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, args):
    return {"workload": wl.name, "d_out": wl.d_out, "d_in": wl.d_in,
            "tokens": wl.n, "bits": wl.bits, "group": wl.group,
            "rot_in": list(wl.rot_in), "rot_out": list(wl.rot_out),
            "l2": "inputs larger than L2 (X alone exceeds 126 MB)",
            "parallelism": f"{args.gpus} independent sublayers, one per GPU"}


# ---------------------------------------------------------------- model stack
def run_stack(args, spec):
    """One step = the whole stack: every covariance and score, the bit
    allocation, every sublayer quantized at its width. Inputs are generated
    per layer on the device (outside the timed spans); the device time is the
    sum of CUDA-event spans around the library calls."""
    import torch

    from second_order_post_b200 import kronq as K
    from second_order_post_b200 import synth
    from second_order_post_b200.stack import StackEngine, device_ms, stack_flops

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("the stack workload runs on one GPU")
    torch.cuda.set_device(0)
    se = StackEngine(spec)
    for _ in range(args.warmup):
        se.run()
    torch.cuda.synchronize()
    se.check_info()
    uuid = "GPU-" + str(torch.cuda.get_device_properties(0).uuid)
    cov_spans, q_spans, totals = [], [], []
    l0 = K.kronq_kernel_launches()
    with ClockSampler(uuid) as clk:
        for _ in range(args.steps):
            c, q = [], []
            for layer in range(spec.layers):
                se.score_layer(layer, timer=c)
            bits = se.allocate()
            S = len(se.HG[0])
            for layer in range(spec.layers):
                for si in range(S):
                    se.quantize_sublayer(layer, si, bits[layer * S + si], timer=q)
            torch.cuda.synchronize()
            cov_spans.append(device_ms(c))
            q_spans.append(device_ms(q))
            totals.append(cov_spans[-1] + q_spans[-1])
    launches = (K.kronq_kernel_launches() - l0) // args.steps
    se.check_info()
    ms = statistics.mean(totals)
    flops = stack_flops(spec)
    n = spec.n
    cov_flops = spec.layers * (sum(n * d * (d + 1) for _, d in synth.STACK_X_GROUPS) +
                               sum(n * do * (do + 1) for _, do, _, _ in synth.STACK_SUBLAYERS))
    peaks, peak_src = load_peaks()
    cov_ms = statistics.mean(cov_spans)
    achieved = cov_flops / (cov_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    hist = [bits.count(b) for b in (2, 3, 4)]
    line = {
        "metric": METRIC, "value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16+f32", "data": "synthetic",
        "config": {"workload": spec.name, "layers": spec.layers,
                   "sublayers": spec.layers * len(synth.STACK_SUBLAYERS),
                   "tokens_per_sublayer": n, "budget_bits": spec.budget,
                   "bits_histogram_2_3_4": hist,
                   "l2": "inputs larger than L2", "parallelism": "1 GPU"},
        "roofline": {"kernel": "cov_bf16 (all covariances of the stack)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16 sustained"},
        "cpu_baseline": None, "e2e": None, "gpu_launches": launches,
        "clocks": clk.summary(),
        "steps_ms": {"covariances_and_scores": cov_ms,
                     "biip_chol_obs_all_sublayers": statistics.mean(q_spans)},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our engine
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()

    from second_order_post_b200 import synth
    if args.workload in synth.STACKS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the oracle arm is timed on the single-sublayer workloads"}))
            return
        run_stack(args, synth.STACKS[args.workload])
        return
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import datetime

    import torch
    import torch.distributed as dist

    from second_order_post_b200 import kronq as K
    from second_order_post_b200.engine import SublayerEngine

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # inputs: one independent sublayer per rank
    wl_r = synth.scaled(wl, seed=wl.seed + 100 * rank)
    data = synth.make_workload(wl_r, device=dev)
    W, X, G = data["W"], data["X"], data["G"]
    eng = SublayerEngine(wl.d_out, wl.d_in, bits=wl.bits, group=wl.group,
                         damp_rel=wl.damp_rel, rot_in=wl.rot_in,
                         rot_out=wl.rot_out, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        eng.run(W, X, G)
    torch.cuda.synchronize()
    eng.check_info()

    names = ["cov_x", "cov_g", "biip", "chol", "quant"]
    marks = []

    def mark(name):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        marks.append((name, e))

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    barrier()
    torch.cuda.synchronize()
    l0 = K.kronq_kernel_launches()
    with ClockSampler(uuid) as clk:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            mark("start")
            eng.run(W, X, G, mark=mark)
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = K.kronq_kernel_launches() - l0
    eng.check_info()
    ms = start.elapsed_time(end) / args.steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    per = {n: [] for n in names}
    for i in range(1, len(marks)):
        if marks[i][0] != "start":
            per[marks[i][0]].append(marks[i - 1][1].elapsed_time(marks[i][1]))
    steps_ms = {n: statistics.mean(v) for n, v in per.items() if v}
    parts, flops = algorithmic_flops(wl)
    value = world * flops / (ms / 1e3) / 1e12

    peaks, peak_src = load_peaks()
    cov_ms = steps_ms["cov_x"]
    achieved = parts["cov_x"] / (cov_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    traffic = load_traffic("cov_bf16", wl.name)
    roofline = {"kernel": "cov_bf16 (H_X = XᵀX/n, tcgen05 bf16)",
                "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "peak_source": f"{peak_src} bf16 sustained"}
    biip_ms = steps_ms["biip"]
    extra = {"biip_gbs": biip_bytes(wl) / (biip_ms / 1e3) / 1e9,
             "biip_hbm_frac": biip_bytes(wl) / (biip_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
             "tensor_frac_cov_plus_quant": (parts["cov_x"] + parts["cov_g"] + parts["quant"])
             / ((steps_ms["cov_x"] + steps_ms["cov_g"] + steps_ms["quant"]) / 1e3) / 1e12 / peak}

    # end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        Wh = W.cpu().pin_memory()
        Xh = X.cpu().pin_memory()
        Gh = G.cpu().pin_memory()
        # two device copies of the inputs: step i+1's copies run under step i
        bufs = [(torch.empty_like(W), torch.empty_like(X), torch.empty_like(G))
                for _ in range(2)]
        codes_h = torch.empty(eng.codes.shape, dtype=eng.codes.dtype, pin_memory=True)
        scales_h = torch.empty(eng.scales.shape, dtype=eng.scales.dtype, pin_memory=True)
        zeros_h = torch.empty(eng.zeros.shape, dtype=eng.zeros.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in (Wh, Xh, Gh))
        d2h = sum(t.numel() * t.element_size() for t in (codes_h, scales_h, zeros_h))
        side = torch.cuda.Stream(device=dev)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        side.wait_event(e0)
        # per buffer set: step name -> event after the step that last read it
        freed = [{}, {}]
        for i in range(args.e2e_steps):
            # the inputs cross on a copy stream, X first, into the buffer set
            # the step before last used; each copy waits only until that
            # step has finished reading the buffer, so the copies of the next
            # sublayer run while this one computes
            Wd, Xd, Gd = bufs[i % 2]
            fr = freed[i % 2]
            arrived = {}
            with torch.cuda.stream(side):
                for key, dst, src in (("cov_x", Xd, Xh), ("cov_g", Gd, Gh), ("biip", Wd, Wh)):
                    if key in fr:
                        side.wait_event(fr[key])
                    dst.copy_(src, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(side)
                    arrived[key] = ev

            def mark(name, fr=fr):
                if name in ("cov_x", "cov_g", "biip"):
                    ev = torch.cuda.Event()
                    ev.record(stream)
                    fr[name] = ev

            eng.run(Wd, Xd, Gd, mark=mark, deps=arrived)
            codes_h.copy_(eng.codes, non_blocking=True)
            scales_h.copy_(eng.scales, non_blocking=True)
            zeros_h.copy_(eng.zeros, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = e0.elapsed_time(e1) / args.e2e_steps
        if world > 1:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": world * flops / (ems / 1e3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": ems, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
        del Wh, Xh, Gh, Wd, Xd, Gd, bufs

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, desc, threads, _ = oracle_sample(wl)
        cpu = {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": threads,
               "kind": "oracle", "sample": desc, "ms_per_sublayer": sec * 1e3,
               "cpu_model": cpu_model(), "nproc": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16+f32", "data": "synthetic",
            "config": workload_config(wl, args), "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk.summary(), "steps_ms": steps_ms, "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
