"""Seeded synthetic sublayer workloads (weights, calibration activations X and
output gradients G) shaped like the LLaMA-2/3 sublayers the KronQ pages
evaluate on.  No trained weights or calibration sets exist here, so these
stand in for them.

This module only draws random inputs: it holds none of the method's
arithmetic and is shared by the tests, the benchmark and the oracle checks so
that both sides of a parity test see identical bytes.

Recipe (per workload; all draws from one ``torch.Generator`` seeded with
``seed``, on the given device):
  W : N(0, 0.02^2) of shape d_out x d_in; ``n_outlier`` seeded input columns
      multiplied by ``outlier_scale`` (LLaMA-style input-dimension outliers).
  X : n x d_in, N(0,1) (or Student-t with 3 degrees of freedom divided by
      sqrt(3)) times a per-channel scale 10^U(x_lo, x_hi).
  G : n x d_out, N(0,1) times a per-channel scale 10^U(g_lo, g_hi); the
      gradient scales span several orders of magnitude, as the pages report
      for H_G's diagonal.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d_out: int
    d_in: int
    n: int
    dtype: torch.dtype
    bits: int
    group: int
    rot_in: tuple
    rot_out: tuple
    n_outlier: int
    outlier_scale: float
    x_range: tuple = (-1.0, 1.0)
    g_range: tuple = (-4.0, 0.0)
    x_student_t: bool = False
    damp_rel: float = 0.01
    seed: int = 0


# Sublayer shapes of the pages' models (LLaMA-2-7B attention and MLP,
# LLaMA-3-70B down_proj).  d = had * m factorisations follow the rotation spec.
WORKLOADS = {
    "small_256": Workload("small_256", 256, 256, 2048, torch.float32, 4, 128,
                          (256, 1), (256, 1), 4, 20.0, (-1.0, 1.0), (-3.0, 0.0)),
    "llama2_7b_attn_4096": Workload("llama2_7b_attn_4096", 4096, 4096, 262144,
                                    torch.bfloat16, 2, 128, (4096, 1),
                                    (4096, 1), 4, 30.0),
    "llama2_7b_mlp_up_11008x4096": Workload(
        "llama2_7b_mlp_up_11008x4096", 11008, 4096, 262144, torch.bfloat16,
        3, 128, (4096, 1), (64, 172), 0, 1.0),
    "llama2_7b_mlp_down_4096x11008": Workload(
        "llama2_7b_mlp_down_4096x11008", 4096, 11008, 262144, torch.bfloat16,
        3, 128, (64, 172), (4096, 1), 0, 1.0, x_student_t=True),
    # 28 outlier columns scaled by 402 give a column CV of |W| near 9.
    "llama3_70b_down_8192x28672": Workload(
        "llama3_70b_down_8192x28672", 8192, 28672, 131072, torch.bfloat16,
        2, 128, (1024, 28), (8192, 1), 28, 402.0),
}


def scaled(w: Workload, **kw) -> Workload:
    """The same workload with some fields replaced (e.g. fewer tokens)."""
    return dataclasses.replace(w, **kw)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def log_uniform(n, lo, hi, gen, device):
    u = torch.rand(n, generator=gen, device=device, dtype=torch.float64)
    return torch.pow(10.0, lo + (hi - lo) * u)


def make_weight(w: Workload, device="cpu", seed=None):
    seed = w.seed + 1000 if seed is None else seed
    gen = _gen(device, seed)
    W = torch.randn(w.d_out, w.d_in, generator=gen, device=device,
                    dtype=torch.float32) * 0.02
    if w.n_outlier:
        cols = torch.randperm(w.d_in, generator=gen, device=device)[:w.n_outlier]
        W[:, cols] *= w.outlier_scale
    return W.to(w.dtype)


def make_activations(n, d, lo, hi, dtype, device="cpu", seed=0,
                     student_t=False, chunk_rows=8192):
    """n x d samples with per-channel log-uniform scales, drawn in row chunks
    so that large bf16 matrices never exist in fp32 in full."""
    gen = _gen(device, seed)
    s = log_uniform(d, lo, hi, gen, device).to(torch.float32)
    out = torch.empty(n, d, dtype=dtype, device=device)
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        z = torch.randn(r1 - r0, d, generator=gen, device=device,
                        dtype=torch.float32)
        if student_t:
            chi = torch.zeros_like(z)
            for _ in range(3):
                e = torch.randn(r1 - r0, d, generator=gen, device=device,
                                dtype=torch.float32)
                chi += e * e
            z = z / torch.sqrt(chi / 3.0) / math.sqrt(3.0)
        out[r0:r1] = (z * s).to(dtype)
    return out


def make_workload(w: Workload, device="cpu", n=None, with_grad=True):
    """Returns dict(W, X, G) for one sublayer; n overrides the token count."""
    n = w.n if n is None else n
    W = make_weight(w, device)
    X = make_activations(n, w.d_in, *w.x_range, w.dtype, device,
                         seed=w.seed + 2000, student_t=w.x_student_t)
    G = make_activations(n, w.d_out, *w.g_range, w.dtype, device,
                         seed=w.seed + 3000) if with_grad else None
    return {"W": W, "X": X, "G": G}


def small_case(d_out, d_in, n, dtype=torch.float32, seed=0, device="cpu",
               n_outlier=2, outlier_scale=20.0):
    """A small random sublayer for unit tests (shapes need not be LLaMA's)."""
    w = Workload("custom", d_out, d_in, n, dtype, 4, 128, (d_in, 1),
                 (d_out, 1), n_outlier, outlier_scale, seed=seed)
    return make_workload(w, device)


def make_spd(d, seed=0, cond_spread=2.0, device="cpu"):
    """A random symmetric positive definite d x d fp32 matrix B Bᵀ/k + diag,
    with log-uniform column scales (for the factorisation tests)."""
    gen = _gen(device, seed)
    k = 2 * d
    b = torch.randn(d, k, generator=gen, device=device, dtype=torch.float64)
    s = log_uniform(d, -cond_spread / 2, cond_spread / 2, gen, device)
    b = b * s[:, None]
    return (b @ b.T / k).to(torch.float32)


# ---------------------------------------------------------------- 7B stack
# A LLaMA-2-7B-shaped stack: per layer the sublayers q, k, v, o (4096 x 4096),
# gate, up (11008 x 4096) and down (4096 x 11008). q, k and v read the same
# input X, and so do gate and up; o and down have their own. Every sublayer
# has its own output gradients G. Each layer draws one scale factor
# 10^U(-1, 1) per tensor kind (W, X, G) that multiplies all of that layer's
# tensors of the kind; within a tensor the recipes of the single-sublayer
# workloads apply (attention W with 4 input columns x30, the down input
# Student-t).
STACK_SUBLAYERS = (
    # name, d_out, d_in, input group
    ("q", 4096, 4096, "attn"),
    ("k", 4096, 4096, "attn"),
    ("v", 4096, 4096, "attn"),
    ("o", 4096, 4096, "o"),
    ("gate", 11008, 4096, "mlp"),
    ("up", 11008, 4096, "mlp"),
    ("down", 4096, 11008, "down"),
)
STACK_X_GROUPS = (("attn", 4096), ("o", 4096), ("mlp", 4096), ("down", 11008))


@dataclasses.dataclass(frozen=True)
class StackSpec:
    name: str = "llama2_7b_stack_224"
    layers: int = 32
    n: int = 32768          # calibration tokens per sublayer
    budget: float = 3.0     # average bits
    group: int = 128
    damp_rel: float = 0.01
    seed: int = 0


STACKS = {"llama2_7b_stack_224": StackSpec()}


def stack_rotation(d):
    """(had, m) of a stack dimension: powers of two rotate with m = 1, 11008
    as Hadamard-64 x Q_172."""
    return (64, 172) if d == 11008 else (d, 1)


def stack_layer_factors(spec: StackSpec, layer: int):
    """(f_W, f_X, f_G): the layer's scale factor per tensor kind."""
    gen = _gen("cpu", spec.seed + 5000 + layer)
    f = torch.pow(10.0, -1.0 + 2.0 * torch.rand(3, generator=gen, dtype=torch.float64))
    return tuple(float(x) for x in f)


def make_stack_x(spec: StackSpec, layer: int, gi: int, device="cpu"):
    name, d = STACK_X_GROUPS[gi]
    fx = stack_layer_factors(spec, layer)[1]
    x = make_activations(spec.n, d, -1.0, 1.0, torch.float32, device,
                         seed=spec.seed + 200000 + 100 * layer + gi,
                         student_t=(name == "down"))
    return (x * fx).to(torch.bfloat16)


def make_stack_g(spec: StackSpec, layer: int, si: int, device="cpu"):
    d_out = STACK_SUBLAYERS[si][1]
    fg = stack_layer_factors(spec, layer)[2]
    g = make_activations(spec.n, d_out, -4.0, 0.0, torch.float32, device,
                         seed=spec.seed + 300000 + 100 * layer + si)
    return (g * fg).to(torch.bfloat16)


def make_stack_w(spec: StackSpec, layer: int, si: int, device="cpu"):
    name, d_out, d_in, group = STACK_SUBLAYERS[si]
    attn = group in ("attn", "o")
    wl = Workload(f"{spec.name}.{layer}.{name}", d_out, d_in, spec.n, torch.bfloat16,
                  2, spec.group, stack_rotation(d_in), stack_rotation(d_out),
                  4 if attn else 0, 30.0 if attn else 1.0)
    fw = stack_layer_factors(spec, layer)[0]
    w = make_weight(wl, device, seed=spec.seed + 100000 + 100 * layer + si)
    return (w.float() * fw).to(torch.bfloat16)
