"""Runs one step of the engine on seeded synthetic inputs, a few times, for
profiling one kernel family with an external profiler:

  python -m second_order_post_b200.run_step cov --d 28672 --n 16384
  python -m second_order_post_b200.run_step biip --workload llama3_70b_down_8192x28672
  python -m second_order_post_b200.run_step matvec --workload llama3_70b_down_8192x28672

cov     kronq_accum_cov on an n x d bf16 X (the sublayer recipe's channel scales)
biip    kronq_biip on the workload's W and on symmetric positive definite
        covariances of its sizes (no covariance pass first)
matvec  kronq_matvec_prepare + kronq_dequant_matvec on random packed codes of
        the workload's shape, one token
chol    kronq_chol_inv on a d x d symmetric positive definite matrix
quant   kronq_chol_inv, then kronq_quantize_sublayer of a d x d weight
        (N(0, 0.02^2)) at 2 bits

Every call goes through the C ABI; the status words are checked at the end.
With --time, each call after the first is timed with CUDA events (L2 flushed
by a 512 MB write before it) and the median is printed in ms.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import kronq as K
from . import synth


class _Timer:
    """Times calls with CUDA events on the current stream, L2 flushed first."""

    def __init__(self, on):
        self.on = on
        self.ms = []
        self.flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device="cuda") if on else None

    def __call__(self, fn, first):
        if not self.on or first:
            fn()
            return
        self.flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        self.ms.append(e0.elapsed_time(e1))


def _spd_like(d, seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    a = torch.randn(d, d, generator=g, device=device) * (0.5 / d ** 0.5)
    a = a + a.T
    a.diagonal().add_(2.0)
    return a


def run_cov(args):
    X = synth.make_activations(args.n, args.d, -1, 1, torch.bfloat16, device="cuda", seed=5)
    H = torch.empty(args.d, args.d, device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r in range(args.reps):
        args.timer(lambda: K.kronq_accum_cov(X, H, 1.0 / args.n, 0.0, info), r == 0)
    torch.cuda.synchronize()
    return [info.item()]


def run_biip(args):
    from .engine import SublayerEngine
    wl = synth.WORKLOADS[args.workload]
    eng = SublayerEngine(wl.d_out, wl.d_in, bits=wl.bits, group=wl.group,
                         rot_in=wl.rot_in, rot_out=wl.rot_out)
    W = synth.make_weight(wl, device="cuda")
    H0x, H0g = _spd_like(wl.d_in, 1, "cuda"), _spd_like(wl.d_out, 2, "cuda")
    for r in range(args.reps):
        eng.H_X.copy_(H0x)
        eng.H_G.copy_(H0g)
        args.timer(lambda: K.kronq_biip(eng.opts, W, eng.W_rot, eng.H_X, eng.H_G, eng.s_x,
                                        eng.s_g, eng.ws, eng.info[2:3]), r == 0)
    torch.cuda.synchronize()
    return [eng.info[2].item()]


def run_matvec(args):
    wl = synth.WORKLOADS[args.workload]
    d_out, d_in, bits = wl.d_out, wl.d_in, wl.bits
    opts = K.make_opts(bits=bits, group=wl.group, rot_in=wl.rot_in, rot_out=wl.rot_out)
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    codes = torch.randint(-2 ** 31, 2 ** 31 - 1, (d_out, bits * d_in // 32), generator=g,
                          dtype=torch.int32, device="cuda")
    scales = torch.rand(d_out, d_in // wl.group, generator=g, device="cuda") * 0.05
    zeros = torch.randint(0, 2 ** bits, (d_out, d_in // wl.group), generator=g,
                          dtype=torch.uint8, device="cuda")
    sx = torch.rand(d_in, generator=g, device="cuda") + 0.5
    sg = torch.rand(d_out, generator=g, device="cuda") + 0.5
    desc = torch.empty(K.kronq_matvec_desc_bytes(opts, d_out, d_in), dtype=torch.uint8,
                       device="cuda")
    K.kronq_matvec_prepare(opts, sx, sg, desc)
    x = torch.randn(1, d_in, generator=g, device="cuda")
    y = torch.empty(1, d_out, device="cuda")
    ws = torch.empty(K.kronq_matvec_workspace_bytes(d_out, d_in, 1), dtype=torch.uint8,
                     device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r in range(args.reps):
        args.timer(lambda: K.kronq_dequant_matvec(opts, desc, codes, scales, zeros, x, y, ws,
                                                  info), r == 0)
    torch.cuda.synchronize()
    return [info.item()]


def run_chol(args):
    from .engine import SublayerEngine
    eng = SublayerEngine(args.d, args.d, bits=2, split=False)
    H0 = _spd_like(args.d, 4, "cuda")
    for r in range(args.reps):
        eng.H_X.copy_(H0)
        args.timer(lambda: K.kronq_chol_inv(eng.H_X, 0.01, eng.ws, eng.info[3:4]), r == 0)
    torch.cuda.synchronize()
    return [eng.info[3].item()]


def run_quant(args):
    from .engine import SublayerEngine
    eng = SublayerEngine(args.d, args.d, bits=2, split=False)
    eng.H_X.copy_(_spd_like(args.d, 4, "cuda"))
    K.kronq_chol_inv(eng.H_X, 0.01, eng.ws, eng.info[3:4])
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    W0 = torch.randn(args.d, args.d, generator=g, device="cuda") * 0.02
    for r in range(args.reps):
        eng.W_rot.copy_(W0)
        args.timer(lambda: K.kronq_quantize_sublayer(eng.opts, eng.W_rot, eng.H_X, eng.codes,
                                                     eng.scales, eng.zeros, eng.ws,
                                                     eng.info[4:5]), r == 0)
    torch.cuda.synchronize()
    return [eng.info[3].item(), eng.info[4].item()]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("step", choices=["cov", "biip", "matvec", "chol", "quant"])
    ap.add_argument("--d", type=int, default=28672)
    ap.add_argument("--n", type=int, default=16384)
    ap.add_argument("--workload", default="llama3_70b_down_8192x28672")
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--time", action="store_true")
    args = ap.parse_args()
    args.timer = _Timer(args.time)
    info = {"cov": run_cov, "biip": run_biip, "matvec": run_matvec, "chol": run_chol,
            "quant": run_quant}[args.step](args)
    if any(info):
        raise SystemExit(f"status word(s) {info}")
    print(f"{args.step} ok")
    if args.time and args.timer.ms:
        shape = ({"workload": args.workload} if args.step in ("biip", "matvec")
                 else {"d": args.d, **({"n": args.n} if args.step == "cov" else {})})
        print(json.dumps({"step": args.step, **shape,
                          "ms_median": statistics.median(args.timer.ms),
                          "timed_calls": len(args.timer.ms)}))


if __name__ == "__main__":
    main()
