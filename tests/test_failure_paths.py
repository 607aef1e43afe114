"""Failure reporting on the GPU, made without any GPU fault.

  - kronq_selftest_timeout: the library's bounded mbarrier wait (the routine
    the covariance and GEMM pipelines wait with) on a barrier that nothing
    completes, under a 1 ms limit. The status word must read
    KRONQ_ERR_TIMEOUT, and the context must stay usable: the next calls on
    the same stream give correct results.
  - a NaN on the diagonal of a covariance: BiIP's diagonal scale and the
    Cholesky step's damping both read the diagonal and must report
    KRONQ_ERR_NONFINITE in their status words.
"""
import numpy as np
import pytest
import torch

import oracle as O
from second_order_post_b200 import synth

pytestmark = pytest.mark.gpu


def _kq():
    from second_order_post_b200 import kronq
    return kronq


def test_wait_that_runs_out_reports_timeout(cuda_device):
    K = _kq()
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        K.kronq_selftest_timeout(1_000_000, info)      # 1 ms
        torch.cuda.synchronize()
        assert info.item() == K.KRONQ_ERR_TIMEOUT
    # the context is still usable: a covariance on the same stream is right
    n, d = 4096, 256
    X = synth.make_activations(n, d, -1, 1, torch.bfloat16, seed=3)
    H = torch.empty(d, d, device="cuda")
    K.kronq_accum_cov(X.cuda(), H, 1.0 / n, 0.0, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    want = O.cov(X.float().numpy())
    got = H.double().cpu().numpy()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) < 1e-4


def test_nan_diagonal_reported_by_biip(cuda_device):
    K = _kq()
    d = 256
    W = torch.randn(d, d, device="cuda") * 0.02
    hx = synth.make_spd(d, seed=1).cuda()
    hg = synth.make_spd(d, seed=2).cuda()
    hx[17, 17] = float("nan")
    opts = K.make_opts(rot_in=(d, 1), rot_out=(d, 1))
    ws = torch.empty(K.kronq_workspace_bytes(K.KRONQ_WS_BIIP, d, d, opts),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty(d, d, device="cuda")
    sx, sg = torch.empty(d, device="cuda"), torch.empty(d, device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kronq_biip(opts, W, out, hx, hg, sx, sg, ws, info)
    torch.cuda.synchronize()
    assert info.item() == K.KRONQ_ERR_NONFINITE


@pytest.mark.parametrize("split", [False, True])
def test_nan_diagonal_reported_by_cholesky(cuda_device, split):
    K = _kq()
    d = 512
    h = synth.make_spd(d, seed=4).cuda()
    h[300, 300] = float("inf") if split else float("nan")
    ws = torch.empty(K.kronq_workspace_bytes(K.KRONQ_WS_CHOL, d, d),
                     dtype=torch.uint8, device="cuda")
    info = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = K.kronq_chol_split if split else K.kronq_chol_inv
    fn(h, 0.01, ws, info)
    torch.cuda.synchronize()
    assert info.item() == K.KRONQ_ERR_NONFINITE
    # a clean factorisation afterwards on the same context
    h = synth.make_spd(d, seed=4).cuda()
    K.kronq_chol_inv(h, 0.01, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
