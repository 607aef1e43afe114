"""Parity at the full sizes of the pages' sublayers, in the launch
configuration the benchmark times: the same C-ABI calls on the same buffers
as SublayerEngine.run, one step at a time so that each step's input can be
kept for the checks. Workloads:
  - LLaMA-3-70B down_proj: W 8192 x 28672, 131072 tokens, W2 g128,
    Hadamard-1024 x Q_28 on the input side;
  - LLaMA-2-7B attention: W 4096 x 4096, 262144 tokens, W2 g128;
  - LLaMA-2-7B MLP gate/up: W 11008 x 4096, 262144 tokens, W3 g128,
    Hadamard-64 x Q_172 on the output side;
  - LLaMA-2-7B MLP down: W 4096 x 11008, 262144 Student-t tokens, W3 g128,
    Hadamard-64 x Q_172 on the input side.

The oracle cannot redo this size in seconds, so the checks are either sampled
outputs it computes one by one or properties that hold at any size:
  H_X, H_G     sampled entries against fp64 dot products of the bf16 columns,
               within 1e-4 of sqrt(H_ii H_jj)
  sensitivity  traces against the fp64 squared norms of X and G (1e-4)
  BiIP         s_x, s_g against the oracle's diagonal scale; Frobenius norms
               and traces preserved; sampled entries of W' and H_X' against
               u_i^T (S M S) u_j with rows u of the rotations built by the
               oracle from the published construction
  U            sampled columns of U^T U (H' + lambda I) against the identity
               (per block in the split form [U11, R12; 0, U22] the engine
               takes for d_in > d_out)
  codes        sampled rows replayed through the oracle's OBS sweep given the
               device's factor (rows are independent given U; in the split
               form, two half sweeps joined through R12)
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from parity_helpers import replay_check
from second_order_post_b200 import synth

pytestmark = pytest.mark.gpu

WORKLOADS = ["llama3_70b_down_8192x28672", "llama2_7b_attn_4096",
             "llama2_7b_mlp_up_11008x4096", "llama2_7b_mlp_down_4096x11008"]


def _rows_matvec(M, v, col_scale=None, row_scale=None, chunk=2048):
    """(diag(row_scale) M diag(col_scale)) @ v in fp64, M on the device in
    row chunks (fp32 or bf16), v an fp64 device vector."""
    out = torch.empty(M.shape[0], dtype=torch.float64, device=M.device)
    for r0 in range(0, M.shape[0], chunk):
        blk = M[r0:r0 + chunk].double()
        if col_scale is not None:
            blk = blk * col_scale[None, :]
        y = blk @ v
        if row_scale is not None:
            y = y * row_scale[r0:r0 + chunk]
        out[r0:r0 + chunk] = y
    return out


@pytest.fixture(scope="module", params=WORKLOADS)
def run(cuda_device, request):
    from second_order_post_b200 import kronq as K
    from second_order_post_b200.engine import SublayerEngine
    torch.cuda.empty_cache()
    wl = synth.WORKLOADS[request.param]
    data = synth.make_workload(wl, device="cuda")
    W, X, G = data["W"], data["X"], data["G"]
    eng = SublayerEngine(wl.d_out, wl.d_in, bits=wl.bits, group=wl.group,
                         damp_rel=wl.damp_rel, rot_in=wl.rot_in, rot_out=wl.rot_out)
    n = X.shape[0]
    K.kronq_accum_cov(X, eng.H_X, 1.0 / n, 0.0, eng.info[0:1])
    K.kronq_accum_cov(G, eng.H_G, 1.0 / n, 0.0, eng.info[1:2])
    K.kronq_sensitivity(eng.H_X, eng.H_G, eng.sens)
    HX0, HG0 = eng.H_X.clone(), eng.H_G.clone()
    K.kronq_biip(eng.opts, W, eng.W_rot, eng.H_X, eng.H_G, eng.s_x, eng.s_g,
                 eng.ws, eng.info[2:3])
    HX1, W1 = eng.H_X.clone(), eng.W_rot.clone()
    if eng.split:   # the engine's choice for this shape (d_in > d_out)
        K.kronq_chol_split(eng.H_X, wl.damp_rel, eng.ws, eng.info[3:4])
        K.kronq_quantize_split(eng.opts, eng.W_rot, eng.H_X, eng.codes, eng.scales,
                               eng.zeros, eng.ws, eng.info[4:5])
    else:
        K.kronq_chol_inv(eng.H_X, wl.damp_rel, eng.ws, eng.info[3:4])
        K.kronq_quantize_sublayer(eng.opts, eng.W_rot, eng.H_X, eng.codes, eng.scales,
                                  eng.zeros, eng.ws, eng.info[4:5])
    torch.cuda.synchronize()
    eng.check_info()
    return dict(wl=wl, W=W, X=X, G=G, eng=eng, HX0=HX0, HG0=HG0, HX1=HX1, W1=W1)


def test_covariance_samples(run):
    rng = np.random.default_rng(1)
    for A, H in ((run["X"], run["HX0"]), (run["G"], run["HG0"])):
        n, d = A.shape
        idx = rng.choice(d, 24, replace=False)
        cols = A[:, torch.as_tensor(idx, device=A.device)].double()
        want = cols.T @ cols / n                     # 24 x 24 exact products
        got = H[torch.as_tensor(idx, device=H.device)][:, torch.as_tensor(idx, device=H.device)].double()
        dg = torch.sqrt(torch.outer(torch.diag(want), torch.diag(want)))
        assert float(((got - want).abs() / dg).max()) <= 1e-4


def test_sensitivity_traces(run):
    eng = run["eng"]
    trs = []
    for A in (run["X"], run["G"]):
        s = 0.0
        for r0 in range(0, A.shape[0], 8192):
            s += float((A[r0:r0 + 8192].double() ** 2).sum())
        trs.append(s / A.shape[0])
    sens = eng.sens.cpu().numpy()
    # the traces inherit the covariances' bar (1e-4): the tensor-core sums of
    # squares keep a drift of a few 1e-5 per accumulator restart
    assert math.isclose(sens[0], trs[0], rel_tol=1e-4)
    assert math.isclose(sens[1], trs[1], rel_tol=1e-4)
    assert math.isclose(sens[2], trs[0] * trs[1], rel_tol=2e-4)


def test_biip_scales_and_invariants(run):
    eng, wl = run["eng"], run["wl"]
    HX0, HG0, HX1, W1 = run["HX0"], run["HG0"], run["HX1"], run["W1"]
    sx = O.diag_scale_of(torch.diag(HX0).double().cpu().numpy(), 0.25)
    sg = O.diag_scale_of(torch.diag(HG0).double().cpu().numpy(), 0.25)
    assert np.abs(eng.s_x.double().cpu().numpy() / sx - 1).max() < 1e-5
    assert np.abs(eng.s_g.double().cpu().numpy() / sg - 1).max() < 1e-5
    s_x, s_g = eng.s_x.double(), eng.s_g.double()
    # ||U_G S_G W S_X U_X^T||_F = ||S_G W S_X||_F
    want = 0.0
    for r0 in range(0, run["W"].shape[0], 2048):
        blk = run["W"][r0:r0 + 2048].double() * s_x[None, :] * s_g[r0:r0 + 2048, None]
        want += float((blk ** 2).sum())
    got = float((W1.double() ** 2).sum())
    assert math.isclose(got, want, rel_tol=1e-5)
    # trace and Frobenius norm of S^-1 H S^-1 survive the rotation
    for H0, H1, s in ((HX0, HX1, s_x), (HG0, run["eng"].H_G, s_g)):
        tr0 = float((torch.diag(H0).double() / s ** 2).sum())
        assert math.isclose(float(torch.diag(H1).double().sum()), tr0, rel_tol=1e-5)
        f0 = 0.0
        for r0 in range(0, H0.shape[0], 2048):
            blk = H0[r0:r0 + 2048].double() / (s[r0:r0 + 2048, None] * s[None, :])
            f0 += float((blk ** 2).sum())
        f1 = 0.0
        for r0 in range(0, H1.shape[0], 2048):
            f1 += float((H1[r0:r0 + 2048].double() ** 2).sum())
        assert math.isclose(f1, f0, rel_tol=1e-5)


def test_biip_sampled_entries(run):
    wl, eng = run["wl"], run["eng"]
    s_x, s_g = eng.s_x.double(), eng.s_g.double()
    W1, HX0, HX1 = run["W1"], run["HX0"], run["HX1"]
    rng = np.random.default_rng(2)
    ux = lambda j: torch.as_tensor(O.rotation_row(0, 0, wl.rot_in[0], wl.rot_in[1], j),
                                   device="cuda")
    ug = lambda i: torch.as_tensor(O.rotation_row(0, 1, wl.rot_out[0], wl.rot_out[1], i),
                                   device="cuda")
    w_rms = float(W1.double().pow(2).mean().sqrt())
    for j in rng.choice(wl.d_in, 3, replace=False):
        y = _rows_matvec(run["W"], ux(int(j)), col_scale=s_x, row_scale=s_g)
        for i in rng.choice(wl.d_out, 3, replace=False):
            want = float(ug(int(i)) @ y)
            assert abs(float(W1[i, j]) - want) <= 1e-5 * w_rms
    for j in rng.choice(wl.d_in, 2, replace=False):
        y = _rows_matvec(HX0, ux(int(j)), col_scale=1 / s_x, row_scale=1 / s_x)
        for i in rng.choice(wl.d_in, 3, replace=False):
            want = float(ux(int(i)) @ y)
            scale = math.sqrt(float(HX1[i, i]) * float(HX1[j, j]))
            assert abs(float(HX1[i, j]) - want) <= 1e-5 * scale


def _inverse_factor_residual(U, Hc, lam, cols, extra=None):
    """max |U^T U (Hc + lambda I) - I| over the sampled columns (U upper,
    Hc symmetric, both fp32 on the device); `extra(c, j)` may modify the
    column of Hc + lambda I first."""
    d = U.shape[0]
    worst = 0.0
    for j in cols:
        c = Hc[:, int(j)].double().clone()
        c[int(j)] += lam
        if extra is not None:
            c = extra(c, int(j))
        y = _rows_matvec(U, c)                       # U c
        z = torch.zeros(d, dtype=torch.float64, device="cuda")
        for r0 in range(0, d, 2048):                 # U^T y
            z += U[r0:r0 + 2048].double().T @ y[r0:r0 + 2048]
        z[int(j)] -= 1.0
        worst = max(worst, float(z.abs().max()))
    return worst


def test_inverse_factor_residual(run):
    """U^T U (H' + lambda I) - I on sampled columns; U comes from fp32
    arithmetic, so the bound is a few units of d * cond * 2^-24. In the split
    form [U11, R12; 0, U22] the checks are per block: U22 against the lower
    right block C, U11 against the Schur complement A - R12 R12^T, and
    R12 = B U22^T on sampled rows."""
    wl, eng, HX1 = run["wl"], run["eng"], run["HX1"]
    F = eng.H_X
    d = F.shape[0]
    assert int(torch.count_nonzero(torch.tril(F[:4096, :4096], -1))) == 0
    lam = wl.damp_rel * float(torch.diag(HX1).double().mean())
    rng = np.random.default_rng(3)
    if not eng.split:
        worst = _inverse_factor_residual(F, HX1, lam, rng.choice(d, 6, replace=False))
        assert worst < 2e-3, worst
        return
    from second_order_post_b200 import kronq as K
    h = K.kronq_chol_split_point(d)
    U11, R12, U22 = F[:h, :h], F[:h, h:], F[h:, h:]
    worst22 = _inverse_factor_residual(U22.contiguous(), HX1[h:, h:].contiguous(), lam,
                                       rng.choice(d - h, 4, replace=False))
    R12c = R12.contiguous()

    def schur(c, j):   # column j of A + lambda I - R12 R12^T
        return c - _rows_matvec(R12c, R12c[j].double())
    worst11 = _inverse_factor_residual(U11.contiguous(), HX1[:h, :h].contiguous(), lam,
                                       rng.choice(h, 4, replace=False), schur)
    assert worst22 < 2e-3, worst22
    assert worst11 < 2e-3, worst11
    U22c = U22.contiguous()
    for i in rng.choice(h, 4, replace=False):       # R12[i] = U22 B[i]^T
        want = _rows_matvec(U22c, HX1[int(i), h:].double())
        got = R12c[int(i)].double()
        assert float((got - want).abs().max()) <= 1e-4 * float(want.abs().max())


def test_codes_sampled_rows(run):
    """Sampled rows replayed through the oracle's OBS sweep given the device's
    factor. In the split form the replay runs in two halves joined through
    R12 (W2 + ((W1 - W_hat1) R12) U22), which the oracle pins show equal to
    the one-pass sweep."""
    wl, eng = run["wl"], run["eng"]
    rows = np.random.default_rng(4).choice(wl.d_out, 6, replace=False)
    ridx = torch.as_tensor(rows, device="cuda")
    w64 = run["W1"][ridx].double().cpu().numpy()
    codes = O.unpack_codes(eng.codes[ridx].cpu().numpy().view(np.uint32), wl.bits, wl.d_in)
    zeros = eng.zeros[ridx].cpu().numpy().astype(np.int64)
    if not eng.split:
        u64 = eng.H_X.double().cpu().numpy()
        ident, n_bad, _ = replay_check(w64, u64, codes, zeros, wl.bits, wl.group)
        assert n_bad == 0
        assert ident >= 0.999
        return
    from second_order_post_b200 import kronq as K
    h = K.kronq_chol_split_point(wl.d_in)
    gh = h // wl.group
    F = eng.H_X
    u11 = F[:h, :h].double().cpu().numpy()
    ident1, bad1, _ = replay_check(w64[:, :h], u11, codes[:, :h], zeros[:, :gh],
                                   wl.bits, wl.group)
    first = O.obs_quantize(w64[:, :h], u11, wl.bits, wl.group,
                           forced_codes=codes[:, :h], forced_zeros=zeros[:, :gh])
    del u11
    r12 = F[:h, h:].double().cpu().numpy()
    p = (w64[:, :h] - first["w_hat"]) @ r12
    del r12
    u22 = F[h:, h:].double().cpu().numpy()
    w2 = w64[:, h:] + p @ u22
    ident2, bad2, _ = replay_check(w2, u22, codes[:, h:], zeros[:, gh:], wl.bits, wl.group)
    assert bad1 == 0 and bad2 == 0
    assert min(ident1, ident2) >= 0.999
