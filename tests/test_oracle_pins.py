"""Pins of the fp64 oracle against facts that do not come from the oracle:
published test vectors, closed forms, invariants the pages state, brute force
on tiny layers and special cases that reduce to textbook routines.

Each test names the passage it follows (page short names as in
include/kronq.h).  All run on CPU (-m "not gpu").
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.stats

import oracle as O
from second_order_post_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _spd(d, seed, spread=2.0):
    return synth.make_spd(d, seed=seed, cond_spread=spread).double().numpy()


# ---------------------------------------------------------------- RNG spec
def test_splitmix64_published_vector():
    want = [int(l, 16) for l in open(os.path.join(GOLDEN, "splitmix64_seed0.txt"))
            if l.startswith("0x")]
    golden = 0x9E3779B97F4A7C15
    states = np.array([(k * golden) % 2 ** 64 for k in range(3)], dtype=np.uint64)
    got = [int(x) for x in O.sm64(states)]
    assert got == want


def test_signs_balanced_and_seeded():
    s0 = O.rotation_signs(0, 0, 1 << 14)
    assert set(np.unique(s0)) == {-1.0, 1.0}
    assert abs(s0.mean()) < 0.03
    assert not np.array_equal(s0, O.rotation_signs(0, 1, 1 << 14))
    assert not np.array_equal(s0, O.rotation_signs(1, 0, 1 << 14))


def test_gaussian_draws_are_standard_normal():
    g = O.gaussian_matrix(7, 0, 256).ravel()
    assert abs(g.mean()) < 0.02 and abs(g.var() - 1) < 0.03
    assert scipy.stats.kstest(g, "norm").pvalue > 1e-3


def _rotation_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "rotation_seed0.txt"))
            if l.strip() and not l.startswith("#")]
    return rows


def test_side_keys_draws_and_signs_seed0():
    # hand-worked values of key = sm64(sm64(seed) + side) and the sign rule
    for row in _rotation_golden():
        kind, side = row[0], int(row[1])
        key = O.side_key(0, side)
        if kind == "key":
            assert int(key) == int(row[2], 16)
        elif kind == "draws":
            got = O.sm64(np.uint64(key) + np.arange(8, dtype=np.uint64))
            assert [int(x) for x in got] == [int(v, 16) for v in row[2:]]
        elif kind == "signs":
            want = [1.0 if c == "+" else -1.0 for c in row[2:]]
            assert O.rotation_signs(0, side, 8).tolist() == want
        elif kind == "kq":
            assert int(key ^ np.uint64(0xA5A5A5A5A5A5A5A5)) == int(row[2], 16)


def test_first_box_muller_normals_seed0():
    # G[0][0] and G[0][1] of each side (counter t = 0, 1), hand-worked
    for row in _rotation_golden():
        if row[0] != "normal":
            continue
        side, t = int(row[1]), int(row[2])
        g = O.gaussian_matrix(0, side, 2)
        assert math.isclose(g[0, t], float(row[7]), rel_tol=1e-13)


def test_diag_scale_hand_examples():
    # floor = 1e-8 * mean of the diagonal as given, then the power
    for line in open(os.path.join(GOLDEN, "diag_scale_examples.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        e, dg, want = (part.split() for part in line.split("|"))
        e = float(e[0])
        dg = np.array([float(x) for x in dg])
        want = np.array([eval(x, {"__builtins__": {}}) for x in want])
        got = O.diag_scale_of(dg, e)
        assert np.allclose(got, want, rtol=1e-13, atol=0)
        assert np.allclose(O.diag_scale(np.diag(dg), e), want, rtol=1e-13, atol=0)


@pytest.mark.parametrize("m", [1, 2, 28, 172])
def test_q_factor_is_the_qr_orthogonal_factor(m):
    q = O.q_factor(3, 1, m)
    assert np.abs(q.T @ q - np.eye(m)).max() < 1e-12
    if m > 1:
        r = q.T @ O.gaussian_matrix(3, 1, m)      # must be R of G = Q R
        assert np.abs(np.tril(r, -1)).max() < 1e-10
        assert (np.diag(r) > 0).all()


def test_hadamard_is_sylvester():
    assert np.allclose(O.hadamard(1), [[1.0]])
    assert np.allclose(O.hadamard(2), np.array([[1, 1], [1, -1]]) / math.sqrt(2))
    for k in range(1, 7):
        h, h2 = O.hadamard(2 ** k), O.hadamard(2 ** (k + 1))
        want = np.block([[h, h], [h, -h]]) / math.sqrt(2)
        assert np.allclose(h2, want, atol=1e-14)
        assert np.abs(h2 @ h2.T - np.eye(2 ** (k + 1))).max() < 1e-12


@pytest.mark.parametrize("had,m", [(256, 1), (64, 4), (4, 28), (2, 172)])
def test_rotation_orthogonal_and_rows(had, m):
    u = O.rotation_matrix(5, 0, had, m)
    assert np.abs(u.T @ u - np.eye(had * m)).max() < 1e-12
    for i in (0, 1, m, had * m - 1):
        assert np.allclose(O.rotation_row(5, 0, had, m, i), u[i], atol=1e-14)


def test_rotation_kron_index_order():
    # (U v)[a*m+b] must be (Hhat · V · Q_mᵀ)[a,b] for V = reshape(sign*v, had x m)
    had, m = 8, 3
    rng = np.random.default_rng(0)
    v = rng.standard_normal(had * m)
    sg = O.rotation_signs(2, 1, had * m)
    want = (O.hadamard(had) @ (sg * v).reshape(had, m) @ O.q_factor(2, 1, m).T).ravel()
    assert np.allclose(O.rotation_matrix(2, 1, had, m) @ v, want)


# ---------------------------------------------------------------- covariances
def test_cov_closed_forms():
    d = 6
    assert np.allclose(O.cov(np.eye(d)), np.eye(d) / d)
    rng = np.random.default_rng(1)
    u, v = rng.standard_normal(10), rng.standard_normal(d)
    assert np.allclose(O.cov(np.outer(u, v)), (u @ u) / 10 * np.outer(v, v))


def test_cov_brute_force():
    rng = np.random.default_rng(2)
    a = rng.standard_normal((5, 3))
    h = O.cov(a)
    for i, j in itertools.product(range(3), range(3)):
        assert math.isclose(h[i, j], math.fsum(a[t, i] * a[t, j] for t in range(5)) / 5,
                            rel_tol=1e-13, abs_tol=1e-15)


# ---------------------------------------------------------------- sensitivity
def test_sensitivity_hand_and_qkv_tie():
    assert O.sensitivity(np.diag([1.0, 2.0]), np.diag([3.0])) == (3.0, 3.0, 9.0)
    x = synth.make_activations(512, 64, -1, 1, synth.torch.float32, seed=1)
    hx = O.cov(x.numpy())
    scores = []
    for s in range(3):  # q, k, v: one X, three gradients
        g = synth.make_activations(512, 64, -4, 0, synth.torch.float32, seed=10 + s)
        scores.append(O.sensitivity(hx, O.cov(g.numpy())))
    assert scores[0][0] == scores[1][0] == scores[2][0]        # tr(H_X) ties
    prods = [s[2] for s in scores]
    assert len(set(prods)) == 3                                  # product separates


# ---------------------------------------------------------------- BiIP
def _layer(d_out, d_in, seed):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((d_out, d_in)) * 0.02
    w[:, rng.choice(d_in, 2, replace=False)] *= 20
    return w, _spd(d_in, seed + 1), _spd(d_out, seed + 2, spread=4.0)


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5])
def test_biip_keeps_kronecker_loss(alpha):
    w, hx, hg = _layer(12, 16, 3)
    wr, hxr, hgr, sx, sg = O.biip(w, hx, hg, seed=4, rot_in=(4, 4),
                                  rot_out=(4, 3), scale_exp=alpha)
    ux, ug = O.rotation_matrix(4, 0, 4, 4), O.rotation_matrix(4, 1, 4, 3)
    rng = np.random.default_rng(5)
    for _ in range(4):
        dw = rng.standard_normal(w.shape)
        dwr = ug @ (sg[:, None] * dw * sx[None, :]) @ ux.T
        a, b = O.layer_loss(dw, hx, hg), O.layer_loss(dwr, hxr, hgr)
        assert abs(a - b) <= 1e-10 * abs(a)
    assert np.allclose(wr, ug @ (sg[:, None] * w * sx[None, :]) @ ux.T)


def test_biip_alpha0_keeps_frobenius_and_traces():
    w, hx, hg = _layer(16, 32, 6)
    wr, hxr, hgr, _, _ = O.biip(w, hx, hg, seed=1, rot_in=(8, 4), scale_exp=0.0)
    assert math.isclose(np.linalg.norm(wr), np.linalg.norm(w), rel_tol=1e-12)
    assert math.isclose(np.trace(hxr), np.trace(hx), rel_tol=1e-12)
    assert math.isclose(np.trace(hgr), np.trace(hg), rel_tol=1e-12)


def test_one_sided_rotations_keep_row_or_column_norms():
    w, hx, hg = _layer(16, 32, 7)
    wi = O.biip(w, hx, hg, seed=2, no_rot_out=True, no_scale=True)[0]
    assert np.allclose(np.linalg.norm(wi, axis=1), np.linalg.norm(w, axis=1))
    assert not np.allclose(np.linalg.norm(wi, axis=0), np.linalg.norm(w, axis=0))
    wo = O.biip(w, hx, hg, seed=2, no_rot_in=True, no_scale=True)[0]
    assert np.allclose(np.linalg.norm(wo, axis=0), np.linalg.norm(w, axis=0))


def test_biip_lowers_cv_on_outliers():
    """wmrh §三 and Q3: on weights with outliers along both dimensions, an
    input-only rotation lowers the column CV but leaves the row CV high, and
    the two-sided BiIP lowers both."""
    data = synth.make_workload(synth.WORKLOADS["small_256"])
    hx, hg = O.cov(data["X"].numpy()), O.cov(data["G"].numpy())
    for seed in range(3):
        rng = np.random.default_rng(seed)
        w = rng.standard_normal((256, 256)) * 0.02
        w[:, rng.choice(256, 8, replace=False)] *= 10
        w[rng.choice(256, 8, replace=False), :] *= 10
        c0, r0 = O.cv_rows_cols(w)
        c1, r1 = O.cv_rows_cols(O.biip(w, hx, hg, seed=0)[0])
        ci, ri = O.cv_rows_cols(O.biip(w, hx, hg, seed=0, no_rot_out=True)[0])
        assert c1 < 0.5 * c0 and r1 < 0.5 * r0
        assert ci < 0.2 * c0 and ri > 0.8 * r0


def test_cv_hand():
    c, r = O.cv_rows_cols(np.array([[1.0, 3.0], [1.0, -3.0]]))
    assert math.isclose(c, 0.5) and r == 0.0


# ---------------------------------------------------------------- Cholesky
def test_chol_inv_identity_and_second_route():
    h = _spd(40, 11)
    u = O.chol_inv(h, 0.01)
    hd = h + O.damping(h, 0.01) * np.eye(40)
    assert np.abs(np.tril(u, -1)).max() == 0 and (np.diag(u) > 0).all()
    assert np.abs(u.T @ u @ hd - np.eye(40)).max() < 1e-10
    # reverse-order Cholesky hd = R Rᵀ (R upper) by flipping, then U = R⁻¹
    j = np.eye(40)[::-1]
    r = j @ np.linalg.cholesky(j @ hd @ j) @ j
    u2 = scipy.linalg.solve_triangular(r, np.eye(40), lower=False)
    assert np.abs(u - u2).max() < 1e-10 * np.abs(u).max()


def test_chol_inv_rejects_indefinite():
    h = np.diag([1.0, 1.0, -5.0, 1.0])
    with pytest.raises(np.linalg.LinAlgError):
        O.chol_inv(h, 0.01)


def test_damping_value():
    assert O.damping(np.diag([1.0, 3.0]), 0.01) == 0.02


# ---------------------------------------------------------------- quantizer / OBS
def test_quant_params_edges():
    s, z, _ = O.quant_params(np.zeros((1, 4)), 2)
    assert s[0] == 1.0 and z[0] == 0.0
    s, z, _ = O.quant_params(np.array([[0.5, 1.5, 3.0]]), 2)       # all positive
    assert math.isclose(s[0], 1.0) and z[0] == 0.0
    s, z, _ = O.quant_params(np.array([[-0.5, -1.5, -3.0]]), 2)    # all negative
    assert math.isclose(s[0], 1.0) and z[0] == 3.0
    s, z, _ = O.quant_params(np.array([[-1.0, 2.0]]), 2)
    assert math.isclose(s[0], 1.0) and z[0] == 1.0
    s, z, zr = O.quant_params(np.array([[-1.0, 2.5]]), 2)    # -xmin/scale = 6/7
    assert math.isclose(zr[0], 6 / 7) and z[0] == 1.0
    s, z, _ = O.quant_params(np.array([[-1.5, 1.5]]), 2)     # 1.5 -> 2 (half to even)
    assert s[0] == 1.0 and z[0] == 2.0
    s, z, _ = O.quant_params(np.array([[-2.5, 0.5]]), 2)     # 2.5 -> 2 (half to even)
    assert s[0] == 1.0 and z[0] == 2.0
    # codes: w = 0.5 with scale 1, zero 2 -> rint(0.5) + 2 = 2 (not 3)
    res = O.rtn_quantize(np.array([[-1.5, 1.5, 0.5, -0.5]]), 2, 4)
    assert list(res["codes"][0]) == [0, 3, 2, 2]


@pytest.mark.parametrize("group", [8, 4])
def test_obs_matches_exact_kronecker_minimiser(group):
    """wmrh §四: with the full Kronecker Hessian H_X ⊗ H_G (H_G dense PD), the
    weights OBS leaves in the still-free columns equal the exact constrained
    minimiser of tr(H_G ΔW H_X ΔWᵀ) given the columns fixed so far, for every
    H_G: so H_G cancels and the U-based update is the OBS optimum."""
    d_out, d_in, bits, damp = 4, 8, 2, 0.01
    rng = np.random.default_rng(21)
    w = rng.standard_normal((d_out, d_in))
    hx, hg = _spd(d_in, 22), _spd(d_out, 23, spread=3.0)
    hxd = hx + O.damping(hx, damp) * np.eye(d_in)
    res = O.obs_quantize(w, O.chol_inv(hx, damp), bits, group)
    k = np.kron(hxd, hg)                                  # column-major vec
    vec = lambda a: a.reshape(-1, order="F")
    for j in range(d_in):
        # columns < j fixed at their quantized values; columns >= j free
        fixed = np.zeros((d_out, d_in), bool)
        fixed[:, :j] = True
        f, fr = vec(fixed), ~vec(fixed)
        delta_fixed = vec(res["w_hat"] - w)[f]
        delta_free = -np.linalg.solve(k[np.ix_(fr, fr)], k[np.ix_(fr, f)] @ delta_fixed)
        state = vec(w)[fr] + delta_free
        col_j = state[:d_out]                             # column j comes first
        gi = j // group
        oracle_col = (res["v"][:, j] - res["zeros"][:, gi]) * res["scales"][:, gi]
        assert np.allclose(col_j, oracle_col, rtol=1e-9, atol=1e-11)


def test_obs_is_rtn_and_bruteforce_when_hessians_diagonal():
    d_out, d_in, bits = 3, 8, 2
    rng = np.random.default_rng(31)
    w = rng.standard_normal((d_out, d_in))
    hx = np.diag(rng.uniform(0.5, 2.0, d_in))
    hg = np.diag(rng.uniform(0.5, 2.0, d_out))
    obs = O.obs_quantize(w, O.chol_inv(hx, 0.0), bits, d_in)
    rtn = O.rtn_quantize(w, bits, d_in)
    assert np.array_equal(obs["codes"], rtn["codes"])
    for r in range(d_out):
        s, z = obs["scales"][r, 0], obs["zeros"][r, 0]
        best = min(itertools.product(range(4), repeat=d_in),
                   key=lambda c: np.sum(np.diag(hx) * (w[r] - s * (np.array(c) - z)) ** 2))
        assert list(obs["codes"][r]) == list(best)
    del hg


def test_obs_between_bruteforce_and_rtn():
    d_out, d_in, bits, damp = 24, 8, 2, 0.01
    rng = np.random.default_rng(41)
    w = rng.standard_normal((d_out, d_in))
    idx = np.arange(d_in)
    hx = 0.9 ** np.abs(idx[:, None] - idx[None, :])      # strongly correlated inputs
    hxd = hx + O.damping(hx, damp) * np.eye(d_in)
    obs = O.obs_quantize(w, O.chol_inv(hx, damp), bits, d_in)
    rtn = O.rtn_quantize(w, bits, d_in)
    cand = np.array(list(itertools.product(range(4), repeat=d_in)), dtype=float)
    l_obs, l_rtn = [], []
    for r in range(d_out):
        s, z = obs["scales"][r, 0], obs["zeros"][r, 0]
        dq = w[r][None, :] - s * (cand - z)
        lb = np.einsum("ij,jk,ik->i", dq, hxd, dq).min()
        lo = (w[r] - obs["w_hat"][r]) @ hxd @ (w[r] - obs["w_hat"][r])
        lr = (w[r] - rtn["w_hat"][r]) @ hxd @ (w[r] - rtn["w_hat"][r])
        assert lb <= lo + 1e-12
        l_obs.append(lo)
        l_rtn.append(lr)
    assert np.mean(l_obs) < 0.8 * np.mean(l_rtn)
    # each decision is the nearest level of the compensated weight
    assert np.array_equal(obs["codes"], np.clip(np.rint(obs["v"]), 0, 3))


def test_obs_many_bits_loss_vanishes():
    rng = np.random.default_rng(51)
    w = rng.standard_normal((6, 16))
    hx, hg = _spd(16, 52), _spd(6, 53)
    u = O.chol_inv(hx, 0.01)
    l2 = O.layer_loss(w - O.obs_quantize(w, u, 2, 16)["w_hat"], hx, hg)
    l16 = O.layer_loss(w - O.obs_quantize(w, u, 16, 16)["w_hat"], hx, hg)
    assert l16 < 1e-7 * l2


def test_obs_forced_replay_reproduces_own_run():
    rng = np.random.default_rng(61)
    w = rng.standard_normal((5, 16))
    u = O.chol_inv(_spd(16, 62), 0.01)
    a = O.obs_quantize(w, u, 3, 8)
    b = O.obs_quantize(w, u, 3, 8, forced_codes=a["codes"], forced_zeros=a["zeros"])
    assert np.array_equal(a["codes"], b["own"]) and np.allclose(a["v"], b["v"])


# ---------------------------------------------------------------- packing
def _read_pack_examples():
    lines = [l.strip() for l in open(os.path.join(GOLDEN, "pack_examples.txt"))
             if l.strip() and not l.startswith("#")]
    for i in range(0, len(lines), 3):
        hdr = dict(kv.split("=") for kv in lines[i].split())
        codes = dict(map(int, kv.split("=")) for kv in lines[i + 1].split())
        words = [int(x, 16) for x in lines[i + 2].split()]
        yield int(hdr["bits"]), int(hdr["d_in"]), codes, words


def test_pack_hand_examples_and_roundtrip():
    for bits, d_in, codes, words in _read_pack_examples():
        c = np.zeros((1, d_in), dtype=np.int64)
        for col, val in codes.items():
            c[0, col] = val
        assert [int(x) for x in O.pack_codes(c, bits)[0]] == words
    rng = np.random.default_rng(71)
    for bits in (2, 3, 4):
        c = rng.integers(0, 2 ** bits, size=(7, 96))
        assert np.array_equal(O.unpack_codes(O.pack_codes(c, bits), bits, 96), c)


# ---------------------------------------------------------------- loss, allocation
def test_layer_loss_is_kronecker_quadratic_form():
    rng = np.random.default_rng(81)
    dw = rng.standard_normal((3, 4))
    hx, hg = _spd(4, 82), _spd(3, 83)
    v = dw.reshape(-1, order="F")
    assert math.isclose(O.layer_loss(dw, hx, hg), v @ np.kron(hx, hg) @ v, rel_tol=1e-12)
    # with H_G = I it is the input-side GPTQ objective summed over rows
    assert math.isclose(O.layer_loss(dw, hx, np.eye(3)),
                        sum(r @ hx @ r for r in dw), rel_tol=1e-12)


@pytest.mark.parametrize("scores,numel,budget,want", [
    ([3, 1, 2], [1, 1, 1], 3.0, [3, 3, 3]),
    ([3, 1, 2], [1, 1, 1], 2.5, [3, 2, 2]),
    ([3, 1, 2], [1, 1, 1], 3.34, [4, 3, 3]),
    ([1, 3, 2], [10, 1, 1], 2.5, [2, 4, 4]),
    ([2, 2, 2], [1, 1, 1], 2.34, [3, 2, 2]),      # tie: lower index first
    ([5, 4], [3, 1], 2.0, [2, 2]),
])
def test_allocator_hand(scores, numel, budget, want):
    assert O.allocate_bits(scores, numel, budget) == want


def test_obs_two_halves_join_through_r12():
    """The GPTQ recursion gives E U = W - W_hat for the scaled errors E, so
    E = (W - W_hat) R with R = U^-1 (H + lambda I = R R^T): the sweep over the
    first h columns reaches the rest only through R12, and running the second
    half from W2 + ((W1 - W_hat1) R12) U22 with U22 reproduces the one-pass
    sweep (same codes, same dequantized weights)."""
    rng = np.random.default_rng(21)
    d_out, d_in, h = 24, 96, 40
    x = rng.standard_normal((3 * d_in, d_in)) @ (np.eye(d_in) + 0.3 * rng.standard_normal((d_in, d_in)) / np.sqrt(d_in))
    x *= np.exp(rng.uniform(-1, 1, d_in))
    hx = x.T @ x / x.shape[0]
    w = rng.standard_normal((d_out, d_in)) * 0.02
    u = O.chol_inv(hx, 0.01)
    r = np.linalg.inv(u)
    for bits, group in ((2, 8), (3, 4), (4, 8)):
        whole = O.obs_quantize(w, u, bits, group)
        first = O.obs_quantize(w[:, :h], u[:h, :h], bits, group)
        w2 = w[:, h:] + ((w[:, :h] - first["w_hat"]) @ r[:h, h:]) @ u[h:, h:]
        second = O.obs_quantize(w2, u[h:, h:], bits, group)
        assert np.array_equal(np.concatenate([first["codes"], second["codes"]], 1), whole["codes"])
        assert np.allclose(np.concatenate([first["w_hat"], second["w_hat"]], 1), whole["w_hat"],
                           atol=1e-12)


# ---------------------------------------------------------------- using the quantized layer
def test_dequantize_hand_examples():
    for line in open(os.path.join(GOLDEN, "dequant_examples.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        bits, sz, codes, want = (part.split() for part in line.split("|"))
        sz = [float(v) for v in sz]
        scales = np.array([sz[0::2]])
        zeros = np.array([sz[1::2]])
        codes = np.array([[int(c) for c in codes]])
        assert max(codes[0]) < 2 ** int(bits[0])
        got = O.dequantize(codes, scales, zeros, 4)
        assert got.tolist() == [[float(v) for v in want]]


@pytest.mark.parametrize("rot_out,rot_in", [((8, 3), (16, 4)), ((32, 1), (64, 1))])
def test_unrotate_matvec_inverts_biip(rot_out, rot_in):
    """W' = U_G S_G W S_X U_Xᵀ from the oracle's BiIP, undone: the sublayer
    applied to x from W' equals W x (orthogonality of U, exact division by
    the scales), for one token and for a batch."""
    d_out, d_in = rot_out[0] * rot_out[1], rot_in[0] * rot_in[1]
    rng = np.random.default_rng(9)
    w = rng.standard_normal((d_out, d_in))
    wr, _, _, sx, sg = O.biip(w, _spd(d_in, 1), _spd(d_out, 2), seed=3,
                              rot_in=rot_in, rot_out=rot_out)
    x = rng.standard_normal((5, d_in))
    y = O.unrotate_matvec(wr, sx, sg, x, seed=3, rot_in=rot_in, rot_out=rot_out)
    assert np.abs(y - x @ w.T).max() < 1e-10 * np.abs(x @ w.T).max()
    y1 = O.unrotate_matvec(wr, sx, sg, x[2], seed=3, rot_in=rot_in, rot_out=rot_out)
    assert np.allclose(y1, y[2], rtol=0, atol=1e-12 * np.abs(y).max())
    # one-sided BiIP (the ablation flags) undone with the same flags
    for fi, fo in ((True, False), (False, True)):
        wr1, _, _, sx1, sg1 = O.biip(w, _spd(d_in, 1), _spd(d_out, 2), seed=3,
                                     rot_in=rot_in, rot_out=rot_out, no_rot_in=fi,
                                     no_rot_out=fo)
        y2 = O.unrotate_matvec(wr1, sx1, sg1, x, seed=3, rot_in=rot_in, rot_out=rot_out,
                               no_rot_in=fi, no_rot_out=fo)
        assert np.abs(y2 - x @ w.T).max() < 1e-10 * np.abs(x @ w.T).max()


def test_dequant_matvec_uses_the_packed_codes():
    """Packed codes, scales and zero points from the OBS sweep reconstruct
    the sweep's own dequantized weights before the rotation is undone."""
    rng = np.random.default_rng(4)
    d_out, d_in, bits, group = 12, 256, 3, 128
    wr = rng.standard_normal((d_out, d_in)) * 0.02
    u = O.chol_inv(_spd(d_in, 5), 0.01)
    res = O.obs_quantize(wr, u, bits, group)
    assert np.array_equal(O.dequantize(res["codes"], res["scales"], res["zeros"], group),
                          res["w_hat"])
    packed = O.pack_codes(res["codes"], bits)
    sx, sg = rng.uniform(0.5, 2.0, d_in), rng.uniform(0.5, 2.0, d_out)
    x = rng.standard_normal(d_in)
    got = O.dequant_matvec(packed, res["scales"], res["zeros"], bits, group, sx, sg, x,
                           seed=1, rot_in=(64, 4), rot_out=(4, 3))
    want = O.unrotate_matvec(res["w_hat"], sx, sg, x, seed=1, rot_in=(64, 4),
                             rot_out=(4, 3))
    assert np.array_equal(got, want)
