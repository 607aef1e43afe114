"""GPU parity: each C-ABI call against the fp64 oracle on identical seeded
inputs (inputs drawn by second_order_post_b200.synth, copied to both sides).

Tolerances (fp32 device arithmetic against an fp64 reference):
  covariances          relative Frobenius error <= 1e-4 (bf16 products are
                       exact in fp32; the error is fp32 accumulation)
  rotated W', H'       relative Frobenius <= 1e-5 (orthogonal transforms of
                       depth log2(d) in fp32: ~log2(d) * 6e-8 per element)
  U (inverse factor)   relative Frobenius <= 2e-4 and |UᵀU(H+λI) - I| <= 1e-3
                       (fp32 Cholesky: forward error ~ cond * d * 6e-8)
  codes                every entry equals the oracle's decision given the
                       same history unless the oracle's pre-rounding value is
                       within 1e-3 of a rounding tie; >= 99.9% identical
  layer loss           relative 1e-3
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from parity_helpers import replay_check
from second_order_post_b200 import synth

pytestmark = pytest.mark.gpu


def K():
    from second_order_post_b200 import kronq
    return kronq


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def dev(x, dtype=None):
    t = torch.as_tensor(x)
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()


# ------------------------------------------------------------------ covariance
# 131072 rows (the 70B down_proj calibration size) and a ragged 139264 run
# over many accumulator restarts; the diagonal (sums of squares, all terms of
# one sign) is where accumulation drift would show first
@pytest.mark.parametrize("n,d", [(64, 128), (1000, 256), (777, 384), (4096, 1024),
                                 (8192, 4096), (131072, 512), (139200, 256)])
def test_cov_bf16(cuda_device, n, d):
    X = synth.make_activations(n, d, -1, 1, torch.bfloat16, seed=n + d)
    H = torch.empty(d, d, device="cuda")
    info = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    K().kronq_accum_cov(X.cuda(), H, 1.0 / n, 0.0, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    want = O.cov(X.float().numpy())
    got = f64(H)
    assert rel_fro(got, want) < 1e-4
    assert np.abs(np.diag(got) / np.diag(want) - 1).max() < 1e-4
    assert torch.equal(H, H.T)                      # both triangles bitwise equal


def test_cov_bf16_accumulates_with_beta(cuda_device):
    n, d = 512, 256
    X1 = synth.make_activations(n, d, -1, 1, torch.bfloat16, seed=1)
    X2 = synth.make_activations(n, d, -1, 1, torch.bfloat16, seed=2)
    H = torch.empty(d, d, device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    K().kronq_accum_cov(X1.cuda(), H, 1.0 / n, 0.0, info)
    K().kronq_accum_cov(X2.cuda(), H, 0.5 / n, 0.5, info)      # mean of two batches
    torch.cuda.synchronize()
    want = O.cov(torch.cat([X1, X2]).float().numpy())
    assert rel_fro(f64(H), want) < 1e-4


@pytest.mark.parametrize("n,d", [(2048, 256), (333, 96)])
def test_cov_f32(cuda_device, n, d):
    X = synth.make_activations(n, d, -1, 1, torch.float32, seed=7)
    H = torch.empty(d, d, device="cuda")
    info = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    K().kronq_accum_cov(X.cuda(), H, 1.0 / n, 0.0, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    assert rel_fro(f64(H), O.cov(X.numpy())) < 1e-5
    assert torch.equal(H, H.T)


def test_sensitivity(cuda_device):
    hx = synth.make_spd(256, seed=1)
    hg = synth.make_spd(384, seed=2, cond_spread=4)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    K().kronq_sensitivity(hx.cuda(), hg.cuda(), out)
    want = O.sensitivity(hx.double().numpy(), hg.double().numpy())
    got = out.tolist()
    for g, w in zip(got, want):
        assert math.isclose(g, w, rel_tol=1e-12)


# ------------------------------------------------------------------ BiIP
BIIP_CASES = [
    # d_out, d_in, rot_out, rot_in, flags, w dtype
    (256, 256, (256, 1), (256, 1), 0, torch.float32),
    (256, 896, (256, 1), (32, 28), 0, torch.float32),
    # 1792 rows of H_X over 148 persistent CTAs: uneven unit counts per CTA
    (1024, 1792, (1024, 1), (64, 28), 0, torch.float32),
    (688, 256, (4, 172), (256, 1), 0, torch.bfloat16),
    (344, 1376, (2, 172), (8, 172), 0, torch.float32),
    (128, 4096, (128, 1), (4096, 1), 0, torch.bfloat16),
    # the fixed-shape row pass (Hadamard-256 x Q_28) and a 4-CTA cluster
    # column pass with the tensor-core Q_28 mix
    (256, 7168, (256, 1), (256, 28), 0, torch.bfloat16),
    (256, 256, (256, 1), (256, 1), 1, torch.float32),
    (256, 256, (256, 1), (256, 1), 2, torch.float32),
    (256, 256, (256, 1), (256, 1), 4, torch.float32),
]


@pytest.mark.parametrize("case", BIIP_CASES)
def test_biip(cuda_device, case):
    Kq = K()
    d_out, d_in, rot_out, rot_in, flags, wdt = case
    data = synth.small_case(d_out, d_in, 1024, seed=d_out + d_in)
    W = data["W"].to(wdt)
    hx = torch.from_numpy(O.cov(data["X"].numpy())).float()
    hg = torch.from_numpy(O.cov(data["G"].numpy())).float()
    opts = Kq.make_opts(seed=3, rot_in=rot_in, rot_out=rot_out, flags=flags)
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_BIIP, d_out, d_in, opts),
                     dtype=torch.uint8, device="cuda")
    Wr = torch.empty(d_out, d_in, device="cuda")
    Hx, Hg = hx.cuda(), hg.cuda()
    sx, sg = torch.empty(d_in, device="cuda"), torch.empty(d_out, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    Kq.kronq_biip(opts, W.cuda(), Wr, Hx, Hg, sx, sg, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    want = O.biip(W.double().numpy(), hx.double().numpy(), hg.double().numpy(),
                  seed=3, rot_in=rot_in, rot_out=rot_out,
                  no_rot_in=bool(flags & 1), no_rot_out=bool(flags & 2),
                  no_scale=bool(flags & 4))
    assert rel_fro(f64(sx), want[3]) < 1e-6
    assert rel_fro(f64(sg), want[4]) < 1e-6
    assert rel_fro(f64(Wr), want[0]) < 1e-5
    assert rel_fro(f64(Hx), want[1]) < 1e-5
    assert rel_fro(f64(Hg), want[2]) < 1e-5


# ------------------------------------------------------------------ Cholesky
# 6016 = 47 blocks of 128: a ragged split whose products (SYRK included) run
# on the 128 x 256 GEMM tiles
@pytest.mark.parametrize("d", [128, 256, 512, 640, 1024, 6016])
def test_chol_inv(cuda_device, d):
    Kq = K()
    h = synth.make_spd(d, seed=d, cond_spread=2.0)
    H = h.cuda()
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_CHOL, d, d),
                     dtype=torch.uint8, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    Kq.kronq_chol_inv(H, 0.01, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    hd = h.double().numpy()
    want = O.chol_inv(hd, 0.01)
    got = f64(H)
    assert np.count_nonzero(np.tril(got, -1)) == 0
    assert rel_fro(got, want) < 2e-4
    lam = O.damping(hd, 0.01)
    resid = got.T @ got @ (hd + lam * np.eye(d)) - np.eye(d)
    assert np.abs(resid).max() < 1e-3


def test_chol_inv_reports_not_pd(cuda_device):
    Kq = K()
    d = 256
    h = synth.make_spd(d, seed=5)
    h[200, 200] = -50.0                     # breaks positive definiteness
    H = h.cuda()
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_CHOL, d, d),
                     dtype=torch.uint8, device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    Kq.kronq_chol_inv(H, 0.0, ws, info)
    torch.cuda.synchronize()
    v = info.item()
    assert v & 0xFF == Kq.KRONQ_ERR_NOT_PD
    assert (v >> 8) >= 200                  # the reverse sweep meets it at or after col 200


# ------------------------------------------------------------------ OBS
def _quant_inputs(d_out, d_in, seed):
    data = synth.small_case(d_out, d_in, 2 * d_in, seed=seed)
    w = data["W"].double().numpy()
    hx = O.cov(data["X"].numpy())
    u = O.chol_inv(hx, 0.01)
    return w.astype(np.float32), u.astype(np.float32)


@pytest.mark.parametrize("d_out,d_in,bits,group", [
    (256, 256, 4, 128), (256, 256, 2, 128), (128, 384, 3, 64),
    (64, 1152, 2, 128), (96, 256, 3, 32)])
def test_quantize(cuda_device, d_out, d_in, bits, group):
    Kq = K()
    w32, u32 = _quant_inputs(d_out, d_in, seed=d_in + bits)
    opts = Kq.make_opts(bits=bits, group=group)
    W = dev(w32)
    codes = torch.empty(d_out, bits * d_in // 32, dtype=torch.int32, device="cuda")
    scales = torch.empty(d_out, d_in // group, device="cuda")
    zeros = torch.empty(d_out, d_in // group, dtype=torch.uint8, device="cuda")
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_QUANT, d_out, d_in, opts),
                     dtype=torch.uint8, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    Kq.kronq_quantize_sublayer(opts, W, dev(u32), codes, scales, zeros, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    got_codes = O.unpack_codes(codes.cpu().numpy().view(np.uint32), bits, d_in)
    got_zeros = zeros.cpu().numpy().astype(np.int64)
    w64, u64 = w32.astype(np.float64), u32.astype(np.float64)
    # free-running comparison (small layers: chains from ties are rare)
    ref = O.obs_quantize(w64, u64, bits, group)
    assert (got_codes == ref["codes"]).mean() >= 0.999
    # decision-by-decision replay: any mismatch must sit at a rounding tie
    ident, n_bad, _ = replay_check(w64, u64, got_codes, got_zeros, bits, group)
    assert n_bad == 0
    assert ident >= 0.999
    # scales and the dequantized weights follow the codes
    rep = O.obs_quantize(w64, u64, bits, group, forced_codes=got_codes,
                         forced_zeros=got_zeros)
    assert rel_fro(f64(scales), rep["scales"]) < 1e-5
    assert rel_fro(f64(W), rep["w_hat"]) < 1e-5


def test_quantize_sampled_rows(cuda_device):
    """A layer large enough for the 128 x 256 GEMM tiles in the trailing
    updates; rows are independent given U, so the oracle checks a sample."""
    Kq = K()
    d_out, d_in, bits, group = 2048, 4096, 2, 128
    data = synth.small_case(d_out, d_in, 2 * d_in, seed=11)
    w32 = data["W"].numpy().astype(np.float32)
    u32 = O.chol_inv(O.cov(data["X"].numpy()), 0.01).astype(np.float32)
    opts = Kq.make_opts(bits=bits, group=group)
    W = dev(w32)
    codes = torch.empty(d_out, bits * d_in // 32, dtype=torch.int32, device="cuda")
    scales = torch.empty(d_out, d_in // group, device="cuda")
    zeros = torch.empty(d_out, d_in // group, dtype=torch.uint8, device="cuda")
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_QUANT, d_out, d_in, opts),
                     dtype=torch.uint8, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    Kq.kronq_quantize_sublayer(opts, W, dev(u32), codes, scales, zeros, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    rows = np.random.default_rng(0).choice(d_out, 48, replace=False)
    got_codes = O.unpack_codes(codes.cpu().numpy().view(np.uint32), bits, d_in)[rows]
    got_zeros = zeros.cpu().numpy().astype(np.int64)[rows]
    w64, u64 = w32[rows].astype(np.float64), u32.astype(np.float64)
    ident, n_bad, _ = replay_check(w64, u64, got_codes, got_zeros, bits, group)
    assert n_bad == 0
    assert ident >= 0.999


# split form: kronq_chol_split + kronq_quantize_split against the one-pass OBS
@pytest.mark.parametrize("d_out,d_in,bits,group", [
    (128, 1024, 2, 128), (96, 1152, 3, 64), (64, 640, 4, 32)])
def test_split_form(cuda_device, d_out, d_in, bits, group):
    Kq = K()
    data = synth.small_case(d_out, d_in, 2 * d_in, seed=d_in + 7 * bits)
    w32 = data["W"].numpy().astype(np.float32)
    hx = O.cov(data["X"].numpy())
    F = dev(hx.astype(np.float32))
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_CHOL, d_out, d_in),
                     dtype=torch.uint8, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    Kq.kronq_chol_split(F, 0.01, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    h = Kq.kronq_chol_split_point(d_in)
    assert h == (d_in // 256) * 128
    # the three blocks against the oracle's U and R = U^-1
    u = O.chol_inv(hx, 0.01)
    r = np.linalg.inv(u)
    f = f64(F)
    assert rel_fro(f[:h, :h], u[:h, :h]) < 2e-4
    assert rel_fro(f[h:, h:], u[h:, h:]) < 2e-4
    assert rel_fro(f[:h, h:], r[:h, h:]) < 2e-4
    assert np.count_nonzero(np.tril(f, -1)) == 0
    opts = Kq.make_opts(bits=bits, group=group)
    W = dev(w32)
    codes = torch.empty(d_out, bits * d_in // 32, dtype=torch.int32, device="cuda")
    scales = torch.empty(d_out, d_in // group, device="cuda")
    zeros = torch.empty(d_out, d_in // group, dtype=torch.uint8, device="cuda")
    qws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_QUANT_SPLIT, d_out, d_in, opts),
                      dtype=torch.uint8, device="cuda")
    Kq.kronq_quantize_split(opts, W, F, codes, scales, zeros, qws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    got_codes = O.unpack_codes(codes.cpu().numpy().view(np.uint32), bits, d_in)
    got_zeros = zeros.cpu().numpy().astype(np.int64)
    w64 = w32.astype(np.float64)
    ref = O.obs_quantize(w64, u, bits, group)
    assert (got_codes == ref["codes"]).mean() >= 0.999
    ident, n_bad, _ = replay_check(w64, u, got_codes, got_zeros, bits, group)
    assert n_bad == 0
    assert ident >= 0.999
    rep = O.obs_quantize(w64, u, bits, group, forced_codes=got_codes, forced_zeros=got_zeros)
    assert rel_fro(f64(W), rep["w_hat"]) < 1e-5


# ------------------------------------------------------------------ GEMM
# (M, N, K, a_mn, b_mn): narrow 128 x 128 tiles, ragged edges, and the wide
# 128 x 256 tiles in every operand major
GEMM_CASES = [(300, 200, 100, 0, 0), (256, 384, 1000, 1, 0), (129, 132, 64, 0, 1),
              (2048, 4096, 4096, 0, 0), (2048, 4096, 1536, 1, 1),
              (1920, 3968, 2080, 0, 1), (4096, 2816, 512, 1, 0)]


@pytest.mark.parametrize("split", ["tf32", "fp16"])
def test_gemm_f32_positive_long_k(cuda_device, split):
    """Sums whose terms all have one sign (a Gram diagonal, as in the
    Cholesky's Schur updates) over a long K: a one-way drift of the
    tensor-core accumulation (up to one unit in the last place per MMA step)
    adds up here instead of cancelling. The main accumulator restarts every
    8192 k and the cross terms accumulate apart, so the drift stays below one
    chunk's steps: (8192 / k-per-MMA) * 2^-23."""
    Kq = K()
    M, N, Kd = 4096, 4096, 16384
    g = torch.Generator(device="cuda").manual_seed(7)
    a = torch.randn(M, Kd, device="cuda", generator=g).abs()
    C = torch.zeros(M, N, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    ws = None
    if split == "fp16":
        ws = torch.empty(Kq.kronq_gemm_f32_workspace_bytes(M, N, Kd), dtype=torch.uint8,
                         device="cuda")
    Kq.kronq_gemm_f32(a, a, C, info, ws=ws)
    torch.cuda.synchronize()
    assert info.item() == 0
    want = a.double() @ a.double().T
    rel = float(((C.double() - want) / want).abs().max())
    kstep = 16 if split == "fp16" else 8
    assert rel < (8192 // kstep) * 2.0 ** -23, rel


@pytest.mark.parametrize("split", ["tf32", "fp16"])
@pytest.mark.parametrize("case", GEMM_CASES)
def test_gemm_f32(cuda_device, case, split):
    """Elementwise against fp64. Each product keeps all but
    1.5 * 2^-20 |a b| (TF32: truncated hi, rounded lo, no lo*lo term; the
    fp16 split of row-scaled operands keeps about 3 * 2^-22) and the
    3K/8 fp32 accumulation steps add rounding that grows like their square
    root: |err| <= (1.5 * 2^-20 + 2 sqrt(3K) 2^-24) |alpha| (|A| |B|^T)
    plus one rounding of the result. A missing or misplaced hi/lo term
    costs ~2^-11 per product and fails this by two orders of magnitude."""
    Kq = K()
    M, N, Kd, a_mn, b_mn = case
    g = torch.Generator(device="cuda").manual_seed(M + N + Kd)
    a = torch.randn(M, Kd, device="cuda", generator=g) * torch.exp(
        torch.randn(1, Kd, device="cuda", generator=g))
    b = torch.randn(N, Kd, device="cuda", generator=g)
    c0 = torch.randn(M, N, device="cuda", generator=g)
    A = a.T.contiguous() if a_mn else a
    B = b.T.contiguous() if b_mn else b
    C = c0.clone()
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    ws = None
    if split == "fp16":   # large products take the fp16 path given a workspace
        ws = torch.empty(Kq.kronq_gemm_f32_workspace_bytes(M, N, Kd), dtype=torch.uint8,
                         device="cuda")
    Kq.kronq_gemm_f32(A, B, C, info, alpha=-0.5, beta=2.0, a_mn=a_mn, b_mn=b_mn, ws=ws)
    torch.cuda.synchronize()
    assert info.item() == 0
    want = 2.0 * c0.double() - 0.5 * (a.double() @ b.double().T)
    rel = 1.5 * 2.0 ** -20 + 2 * math.sqrt(3 * Kd) * 2.0 ** -24
    bound = rel * 0.5 * (a.double().abs() @ b.double().abs().T) + \
        2.0 ** -23 * want.abs() + 1e-30
    err = (C.double() - want).abs()
    assert bool((err <= bound).all()), float((err / bound).max())


# ------------------------------------------------------------------ loss
@pytest.mark.parametrize("d_out,d_in", [(256, 384), (2048, 4096)])
def test_layer_loss(cuda_device, d_out, d_in):
    Kq = K()
    rng = np.random.default_rng(3)
    a = rng.standard_normal((d_out, d_in)).astype(np.float32)
    b = (a + 0.01 * rng.standard_normal((d_out, d_in))).astype(np.float32)
    hx = synth.make_spd(d_in, seed=4)
    hg = synth.make_spd(d_out, seed=5, cond_spread=4)
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.empty(Kq.kronq_workspace_bytes(Kq.KRONQ_WS_LOSS, d_out, d_in),
                     dtype=torch.uint8, device="cuda")
    info = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    Kq.kronq_layer_loss(dev(a), dev(b), hx.cuda(), hg.cuda(), loss, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    want = O.layer_loss(a.astype(np.float64) - b, hx.double().numpy(), hg.double().numpy())
    # error budget of the two fp32-accurate products P = D H_X, Q = H_G D
    # (per element as in test_gemm_f32) carried through sum(P * Q)
    dd = torch.from_numpy(a.astype(np.float64) - b).cuda()
    hxd, hgd = hx.double().cuda(), hg.double().cuda()
    P, Q = dd @ hxd, hgd @ dd
    rel = lambda k: 1.5 * 2.0 ** -20 + 2 * math.sqrt(3 * k) * 2.0 ** -24 + 2.0 ** -23
    bound = rel(d_in) * float(((dd.abs() @ hxd.abs()) * Q.abs()).sum()) + \
        rel(d_out) * float((P.abs() * (hgd.abs() @ dd.abs())).sum())
    assert abs(loss.item() - want) <= bound
    assert math.isclose(loss.item(), want, rel_tol=1e-3)   # the method's bar
