"""Every entry of the rotated H_X at the Hadamard ⊗ Q_28 shapes of the pages'
70B MLP (d_in = 1024 * 28 = 28672) and of a half-size 512 * 28 = 14336,
against an fp64 reference built from the oracle's factors.

The oracle's dense U = (Hhat ⊗ Q_m) diag(sign) (oracle.rotation_matrix) is
6.6 GB at d = 28672 and U H Uᵀ takes 9.4e13 flop, so the reference applies
the same factors (oracle.hadamard, oracle.q_factor, oracle.rotation_signs,
oracle.diag_scale_of) one Kronecker factor at a time with fp64 torch matmuls
on the device:
    M  = diag(sign/s) H diag(sign/s)
    M <- (Hhat ⊗ Q) M (Hhat ⊗ Q)ᵀ     (Hhat on the a axes, Q on the b axes)
where index i = a*m + b. The BiIP kernels of these shapes are the row pass
over rows held in shared memory two at a time (the next row's bulk copy in
flight) and, at 28672, the column pass over 16-CTA clusters.
Bar: relative Frobenius error <= 1e-5 (as the small BiIP cases) and every
entry within 1e-5 of max |H'| (fp32 transforms of depth ~log2(d)).
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

SEED = 3


def _reference(H, had, m, seed=SEED):
    d = had * m
    diag = H.diagonal().double().cpu().numpy()
    s = O.diag_scale_of(diag, 0.25)
    f = torch.from_numpy(O.rotation_signs(seed, 0, d) / s).cuda()
    Hd = torch.from_numpy(O.hadamard(had)).cuda()
    Q = torch.from_numpy(O.q_factor(seed, 0, m)).cuda()
    M = H.double() * f[:, None] * f[None, :]
    # rows: i = (a, b) -> (Hhat ⊗ Q) from the left
    M = (Hd @ M.view(had, m * d)).view(had, m, d)
    M = torch.matmul(Q, M).view(d, d)
    # columns: the same factors from the right
    M = torch.matmul(M.view(d, had, m), Q.T)
    M = torch.matmul(Hd, M).view(d, d)
    return M, s


@pytest.mark.parametrize("had", [1024, 512])
def test_biip_hx_every_entry(cuda_device, had):
    from second_order_post_b200 import kronq as K
    m, d_out = 28, 256
    d = had * m
    g = torch.Generator(device="cuda")
    g.manual_seed(had)
    A = torch.randn(d, d, generator=g, device="cuda")
    H = (A + A.T) * 0.5
    del A
    H.diagonal().abs_().add_(1.0)
    want, s_want = _reference(H, had, m)
    W = torch.randn(d_out, d, generator=g, device="cuda") * 0.02
    Hg = torch.eye(d_out, device="cuda") * 2.0
    opts = K.make_opts(seed=SEED, rot_in=(had, m), rot_out=(d_out, 1))
    ws = torch.empty(K.kronq_workspace_bytes(K.KRONQ_WS_BIIP, d_out, d, opts),
                     dtype=torch.uint8, device="cuda")
    Wr = torch.empty(d_out, d, device="cuda")
    sx, sg = torch.empty(d, device="cuda"), torch.empty(d_out, device="cuda")
    info = torch.ones(1, dtype=torch.int32, device="cuda")
    K.kronq_biip(opts, W, Wr, H, Hg, sx, sg, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    assert np.abs(sx.double().cpu().numpy() / s_want - 1).max() < 1e-6
    err = (H.double() - want)
    scale = want.abs().max()
    rel = float(torch.linalg.norm(err) / torch.linalg.norm(want))
    worst = float(err.abs().max() / scale)
    assert rel < 1e-5, rel
    assert worst < 1e-5, worst
