"""Plain fp64 CPU oracle of the KronQ per-sublayer quantization engine.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never
imports, links or calls it, and this module imports nothing from the product.

Every function is the plainest reading of the pages about arXiv 2607.07964
("KronQ: LLM Quantization via Kronecker-Factored Hessian"), in float64, with
library primitives (matmul, QR, Cholesky, inverse) as single steps and no
blocking or reordering beyond what the method states.  Sources are cited by
the short names used in ``include/kronq.h``:

  [gptget-en]  gptget.net English summary (Methodology, Technical Contribution)
  [aimodeling] aimodeling.com news "KronQ: Kronecker Hessians break GPTQ's
               2-bit wall" (H ≈ H_X ⊗ H_G; BiIP; tr(H_G)·tr(H_X))
  [wmrh]       wmrh.cn article, sections 二 (Kronecker Hessian), 三 (BiIP,
               sensitivity), 四 (H_G cancels from the column update), 五
               (W2/W3/W4, g128), 六 (mixed precision), 七 (H_G freed after
               preprocessing), 八 (S_X/S_G diagonal scaling before rotation)

Where the pages leave a step open, the reading used here is the one written
out in ``include/kronq.h`` (rotation/RNG spec, quantizer edge cases).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, brute force or published test vectors.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "sm64", "rotation_signs", "gaussian_matrix", "q_factor", "hadamard",
    "rotation_matrix", "diag_scale", "cov", "sensitivity", "biip",
    "damping", "chol_inv", "quant_params", "obs_quantize", "rtn_quantize",
    "pack_codes", "unpack_codes", "layer_loss", "cv_rows_cols",
    "allocate_bits", "dequantize", "unrotate_matvec", "dequant_matvec",
]

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)
_QKEY = np.uint64(0xA5A5A5A5A5A5A5A5)


# --------------------------------------------------------------------------
# splitmix64 and the rotation spec (include/kronq.h, "Rotation and
# random-number specification")
# --------------------------------------------------------------------------
def sm64(s):
    """splitmix64 output for state ``s`` (array of uint64, wraps mod 2^64).

    Published definition (Steele, Lea & Flood 2014; Vigna's reference C):
    z = s + golden; z = (z ^ z>>30) * c1; z = (z ^ z>>27) * c2; z ^ z>>31.
    """
    z = np.asarray(s, dtype=np.uint64) + _GOLDEN
    z = (z ^ (z >> np.uint64(30))) * _MIX1
    z = (z ^ (z >> np.uint64(27))) * _MIX2
    return z ^ (z >> np.uint64(31))


def side_key(seed: int, side: int) -> np.ndarray:
    """key = sm64(sm64(seed) + side); side 0 = input (d_in), 1 = output."""
    k0 = sm64(np.array([seed], dtype=np.uint64))
    return sm64(k0 + np.uint64(side))[0]


def rotation_signs(seed: int, side: int, d: int) -> np.ndarray:
    """±1 diagonal: +1 when bit 63 of sm64(key + i) is clear."""
    key = side_key(seed, side)
    h = sm64(key + np.arange(d, dtype=np.uint64))
    return np.where((h >> np.uint64(63)) == 0, 1.0, -1.0)


def gaussian_matrix(seed: int, side: int, m: int) -> np.ndarray:
    """m x m Box–Muller normals from splitmix64 counters (one normal per pair)."""
    kq = side_key(seed, side) ^ _QKEY
    t = np.arange(m * m, dtype=np.uint64)
    x1 = sm64(kq + np.uint64(2) * t)
    x2 = sm64(kq + np.uint64(2) * t + np.uint64(1))
    u1 = ((x1 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (x2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return g.reshape(m, m)


def q_factor(seed: int, side: int, m: int) -> np.ndarray:
    """Orthogonal factor of G = Q R with R[j][j] > 0 (unique)."""
    if m == 1:
        return np.ones((1, 1))
    g = gaussian_matrix(seed, side, m)
    q, r = np.linalg.qr(g)
    d = np.sign(np.diag(r))
    d[d == 0] = 1.0
    return q * d[None, :]


def hadamard(had: int) -> np.ndarray:
    """Normalised Sylvester Hadamard: entries (-1)^popcount(a & a') / sqrt(had)."""
    a = np.arange(had)
    bits = np.bitwise_and.outer(a, a)
    pc = np.zeros_like(bits)
    while bits.any():
        pc += bits & 1
        bits >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0) / math.sqrt(had)


def rotation_matrix(seed: int, side: int, had: int, m: int) -> np.ndarray:
    """Dense U = (Hhat ⊗ Q_m) · diag(sign) of size (had*m)^2 [wmrh §三, Q2]."""
    d = had * m
    u = np.kron(hadamard(had), q_factor(seed, side, m))
    return u * rotation_signs(seed, side, d)[None, :]


def rotation_row(seed: int, side: int, had: int, m: int, i: int) -> np.ndarray:
    """Row i of U without forming U (for sampled checks at large d)."""
    a, b = divmod(i, m)
    ap = np.arange(had)
    bits = np.bitwise_and(ap, a)
    pc = np.zeros_like(bits)
    while bits.any():
        pc += bits & 1
        bits >>= 1
    hrow = np.where(pc % 2 == 0, 1.0, -1.0) / math.sqrt(had)
    qrow = q_factor(seed, side, m)[b]
    return np.kron(hrow, qrow) * rotation_signs(seed, side, had * m)


# --------------------------------------------------------------------------
# Step 1: covariances [wmrh §二; aimodeling]
# --------------------------------------------------------------------------
def cov(a: np.ndarray) -> np.ndarray:
    """H = Aᵀ A / n over the n calibration rows of A (n x d), in fp64."""
    a = np.asarray(a, dtype=np.float64)
    return a.T @ a / a.shape[0]


# --------------------------------------------------------------------------
# Step 2: sensitivity [wmrh §三, §六; aimodeling]
# --------------------------------------------------------------------------
def sensitivity(h_x: np.ndarray, h_g: np.ndarray):
    """(tr H_X, tr H_G, tr H_G · tr H_X) on the un-rotated, un-scaled H."""
    tx = float(np.trace(np.asarray(h_x, dtype=np.float64)))
    tg = float(np.trace(np.asarray(h_g, dtype=np.float64)))
    return tx, tg, tx * tg


# --------------------------------------------------------------------------
# Step 3: BiIP [wmrh §三, §八; aimodeling]
# --------------------------------------------------------------------------
def diag_scale(h: np.ndarray, exponent: float) -> np.ndarray:
    """s_i = max(h_ii, 1e-8·mean(diag h))^exponent (reading of wmrh §八)."""
    return diag_scale_of(np.diag(np.asarray(h, dtype=np.float64)), exponent)


def diag_scale_of(dg: np.ndarray, exponent: float) -> np.ndarray:
    """diag_scale from the diagonal alone (for sizes where H is not kept)."""
    dg = np.asarray(dg, dtype=np.float64).copy()
    floor = 1e-8 * dg.mean()
    return np.maximum(dg, floor) ** exponent


def biip(w, h_x, h_g, seed=0, rot_in=None, rot_out=None, scale_exp=0.25,
         no_rot_in=False, no_rot_out=False, no_scale=False):
    """Two-sided rescale + rotation.

    Returns (W', H_X', H_G', s_x, s_g) with
      W'   = U_G S_G W S_X U_Xᵀ
      H_X' = U_X S_X⁻¹ H_X S_X⁻¹ U_Xᵀ,   H_G' = U_G S_G⁻¹ H_G S_G⁻¹ U_Gᵀ.
    rot_in / rot_out are (had, m) pairs; default (d, 1).
    """
    w = np.asarray(w, dtype=np.float64)
    h_x = np.asarray(h_x, dtype=np.float64)
    h_g = np.asarray(h_g, dtype=np.float64)
    d_out, d_in = w.shape
    rot_in = rot_in or (d_in, 1)
    rot_out = rot_out or (d_out, 1)
    if no_scale:
        s_x, s_g = np.ones(d_in), np.ones(d_out)
    else:
        s_x, s_g = diag_scale(h_x, scale_exp), diag_scale(h_g, scale_exp)
    u_x = np.eye(d_in) if no_rot_in else rotation_matrix(seed, 0, *rot_in)
    u_g = np.eye(d_out) if no_rot_out else rotation_matrix(seed, 1, *rot_out)
    w_rot = u_g @ (s_g[:, None] * w * s_x[None, :]) @ u_x.T
    hx_rot = u_x @ (h_x / np.outer(s_x, s_x)) @ u_x.T
    hg_rot = u_g @ (h_g / np.outer(s_g, s_g)) @ u_g.T
    return w_rot, hx_rot, hg_rot, s_x, s_g


# --------------------------------------------------------------------------
# Step 4: damped inverse Cholesky factor [wmrh §四]
# --------------------------------------------------------------------------
def damping(h: np.ndarray, damp_rel: float) -> float:
    """lambda = damp_rel · mean(diag H)."""
    return float(damp_rel * np.mean(np.diag(np.asarray(h, dtype=np.float64))))


def chol_inv(h: np.ndarray, damp_rel: float) -> np.ndarray:
    """Upper U with Uᵀ U = (H + λI)⁻¹: dense inverse, then Cholesky of it.

    Raises numpy.linalg.LinAlgError when H + λI is not positive definite.
    """
    h = np.asarray(h, dtype=np.float64)
    hd = h + damping(h, damp_rel) * np.eye(h.shape[0])
    lower = np.linalg.cholesky(hd)                  # hd = L Lᵀ
    eye = np.eye(h.shape[0])
    hinv = np.linalg.solve(lower.T, np.linalg.solve(lower, eye))
    hinv = 0.5 * (hinv + hinv.T)
    return np.linalg.cholesky(hinv).T               # hinv = Lᵢ Lᵢᵀ = Uᵀ U


# --------------------------------------------------------------------------
# Step 5: quantizer and column-wise OBS [gptget-en Methodology; wmrh §四, §五]
# --------------------------------------------------------------------------
def quant_params(wg: np.ndarray, bits: int):
    """Asymmetric min-max (scale, zero) per row of the group slice ``wg``."""
    maxq = 2 ** bits - 1
    xmin = np.minimum(wg.min(axis=1), 0.0)
    xmax = np.maximum(wg.max(axis=1), 0.0)
    flat = xmax == xmin
    scale = np.where(flat, 1.0, (xmax - xmin) / maxq)
    zero = np.where(flat, 0.0, np.rint(-xmin / scale))
    return scale, zero, -xmin / np.where(flat, 1.0, scale)


def obs_quantize(w, u, bits: int, group: int, forced_codes=None,
                 forced_zeros=None):
    """Column-by-column OBS sweep with the full trailing update per column.

    For j = 0 .. d_in-1 (all rows at once; rows never interact, [wmrh §四]):
      at a group start: (scale, zero) from the row's current weights of the
      group; q = clamp(rint(w_j/scale) + zero, 0, 2^b-1);
      w_hat = scale·(q - zero); err = (w_j - w_hat)/U[j,j];
      W[:, j+1:] -= err ⊗ U[j, j+1:].

    ``forced_codes`` (same shape as W, optional) replays a candidate's
    decisions: the sweep then follows the given codes instead of its own,
    while still reporting its own pre-rounding values ``v`` and decisions.
    ``forced_zeros`` likewise replaces the zero points (shape d_out x groups).
    This lets a caller check that every decision of a candidate is the
    correctly rounded one given the candidate's own earlier choices.

    Returns dict with codes (int64), w_hat, scales, zeros, v (w/scale + zero
    before rounding), zraw (-xmin/scale before rounding), own (own decisions).
    """
    w = np.array(w, dtype=np.float64, copy=True)
    u = np.asarray(u, dtype=np.float64)
    d_out, d_in = w.shape
    maxq = 2 ** bits - 1
    ng = d_in // group
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    own = np.zeros((d_out, d_in), dtype=np.int64)
    v_all = np.zeros((d_out, d_in))
    w_hat = np.zeros((d_out, d_in))
    scales = np.zeros((d_out, ng))
    zeros = np.zeros((d_out, ng))
    zraw = np.zeros((d_out, ng))
    scale = zero = None
    for j in range(d_in):
        if j % group == 0:
            gi = j // group
            scale, zero, zr = quant_params(w[:, j:j + group], bits)
            if forced_zeros is not None:
                zero = np.asarray(forced_zeros[:, gi], dtype=np.float64)
            scales[:, gi], zeros[:, gi], zraw[:, gi] = scale, zero, zr
        v = w[:, j] / scale + zero
        q_own = np.clip(np.rint(w[:, j] / scale) + zero, 0, maxq)
        q = q_own if forced_codes is None else \
            np.asarray(forced_codes[:, j], dtype=np.float64)
        wh = scale * (q - zero)
        err = (w[:, j] - wh) / u[j, j]
        w[:, j + 1:] -= np.outer(err, u[j, j + 1:])
        v_all[:, j], own[:, j], codes[:, j], w_hat[:, j] = v, q_own, q, wh
    return {"codes": codes, "w_hat": w_hat, "scales": scales, "zeros": zeros,
            "v": v_all, "zraw": zraw, "own": own}


def rtn_quantize(w, bits: int, group: int):
    """Round-to-nearest with the same group quantizer (OBS with U = I)."""
    return obs_quantize(w, np.eye(np.asarray(w).shape[1]), bits, group)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Little-endian bitstream per row: code of column c in bits [c·b, c·b+b)."""
    codes = np.asarray(codes, dtype=np.int64)
    d_out, d_in = codes.shape
    nw = bits * d_in // 32
    out = np.zeros((d_out, nw), dtype=np.uint64)
    for c in range(d_in):
        for t in range(bits):
            pos = c * bits + t
            bit = ((codes[:, c] >> t) & 1).astype(np.uint64)
            out[:, pos // 32] |= bit << np.uint64(pos % 32)
    return out.astype(np.uint32)


def unpack_codes(words: np.ndarray, bits: int, d_in: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint64)
    out = np.zeros((words.shape[0], d_in), dtype=np.int64)
    for c in range(d_in):
        for t in range(bits):
            pos = c * bits + t
            bit = (words[:, pos // 32] >> np.uint64(pos % 32)) & np.uint64(1)
            out[:, c] |= bit.astype(np.int64) << t
    return out


# --------------------------------------------------------------------------
# Using the quantized sublayer: dequantize, undo the two-sided rotation
# [aimodeling: packed low-bit weights with a fused dequant + BiIP matvec;
# wmrh Q2: two Hadamard transforms per layer at inference]
# --------------------------------------------------------------------------
def dequantize(codes, scales, zeros, group: int) -> np.ndarray:
    """The quantizer's reconstruction: w_hat[i, c] = scale[i, g]·(q[i, c] −
    zero[i, g]) with g = c // group (codes unpacked, d_out x d_in)."""
    codes = np.asarray(codes, dtype=np.float64)
    g = np.arange(codes.shape[1]) // group
    scales = np.asarray(scales, dtype=np.float64)
    zeros = np.asarray(zeros, dtype=np.float64)
    return scales[:, g] * (codes - zeros[:, g])


def unrotate_matvec(w_rot, s_x, s_g, x, seed=0, rot_in=None, rot_out=None,
                    no_rot_in=False, no_rot_out=False):
    """y = W x for the sublayer whose rotated weights are W' = U_G S_G W S_X
    U_Xᵀ, i.e. y = S_G⁻¹ U_Gᵀ W' U_X S_X⁻¹ x, with dense rotations built
    from the spec (a side without rotation, as in biip's flags, has U = I).
    x is d_in (one token) or B x d_in (one token per row)."""
    w_rot = np.asarray(w_rot, dtype=np.float64)
    d_out, d_in = w_rot.shape
    rot_in = rot_in or (d_in, 1)
    rot_out = rot_out or (d_out, 1)
    u_x = np.eye(d_in) if no_rot_in else rotation_matrix(seed, 0, *rot_in)
    u_g = np.eye(d_out) if no_rot_out else rotation_matrix(seed, 1, *rot_out)
    xt = np.atleast_2d(np.asarray(x, dtype=np.float64)).T          # d_in x B
    x1 = xt / np.asarray(s_x, dtype=np.float64)[:, None]
    y = u_g.T @ (w_rot @ (u_x @ x1))
    y = y / np.asarray(s_g, dtype=np.float64)[:, None]
    return y.T if np.ndim(x) == 2 else y[:, 0]


def dequant_matvec(packed, scales, zeros, bits: int, group: int, s_x, s_g, x,
                   seed=0, rot_in=None, rot_out=None):
    """The quantized sublayer applied to x: unpack, dequantize, undo the
    rotation."""
    packed = np.asarray(packed)
    d_in = packed.shape[1] * 32 // bits
    w_hat = dequantize(unpack_codes(packed, bits, d_in), scales, zeros, group)
    return unrotate_matvec(w_hat, s_x, s_g, x, seed, rot_in, rot_out)


# --------------------------------------------------------------------------
# Measurement: Kronecker loss and coefficient of variation
# --------------------------------------------------------------------------
def layer_loss(dw, h_x, h_g) -> float:
    """tr(H_G ΔW H_X ΔWᵀ) = vec(ΔW)ᵀ (H_X ⊗ H_G) vec(ΔW) [aimodeling; wmrh §二]."""
    dw = np.asarray(dw, dtype=np.float64)
    return float(np.sum((np.asarray(h_g, dtype=np.float64) @ dw) *
                        (dw @ np.asarray(h_x, dtype=np.float64))))


def cv_rows_cols(w):
    """Coefficient of variation (population std / mean) of the column means
    and the row means of |W| [wmrh §三 "变异系数"]. Returns (cv_col, cv_row)."""
    a = np.abs(np.asarray(w, dtype=np.float64))
    c, r = a.mean(axis=0), a.mean(axis=1)
    return float(c.std() / c.mean()), float(r.std() / r.mean())


# --------------------------------------------------------------------------
# Mixed-precision allocation [wmrh §六]
# --------------------------------------------------------------------------
def allocate_bits(scores, numel, avg_budget: float):
    """Greedy: start at 2 bits; upgrade 2→3, then 3→4, in descending score
    (ties: lower index first), keeping the parameter-weighted mean ≤ budget."""
    scores = [float(s) for s in scores]
    numel = [int(x) for x in numel]
    n = len(scores)
    total = float(sum(numel))
    bits = [2] * n
    used = 2.0 * total
    order = sorted(range(n), key=lambda i: (-scores[i], i))
    for frm in (2, 3):
        for i in order:
            if bits[i] == frm and used + numel[i] <= avg_budget * total:
                bits[i] = frm + 1
                used += numel[i]
    return bits
