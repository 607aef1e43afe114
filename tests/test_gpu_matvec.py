"""kronq_dequant_matvec: the quantized sublayer applied to activations,
y = S_G^-1 U_G^T W_hat' U_X S_X^-1 x, against the oracle's dense fp64
reconstruction (unpack, dequantize, dense rotations from the spec).

Tolerance: y1 = W_hat' x2 sums d_in fp32 products and the two rotations add
log2(d) fp32 rounds; the relative Frobenius error of y is held to 2e-5."""
import numpy as np
import pytest
import torch

import oracle as O
from second_order_post_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    # d_out, d_in, rot_out, rot_in, bits, group, n_tokens, flags
    (256, 256, (256, 1), (256, 1), 4, 128, 1, 0),
    (384, 896, (128, 3), (32, 28), 2, 128, 3, 0),
    (688, 1376, (4, 172), (8, 172), 3, 32, 2, 0),
    (256, 512, (256, 1), (512, 1), 2, 64, 2, 1),
    (256, 512, (256, 1), (512, 1), 2, 64, 1, 2),
    (4096, 7168, (4096, 1), (256, 28), 2, 128, 1, 0),
]


def _kq():
    from second_order_post_b200 import kronq
    return kronq


def _random_layer(d_out, d_in, bits, group, seed):
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 2 ** bits, (d_out, d_in), generator=g).numpy()
    scales = (torch.rand(d_out, d_in // group, generator=g, dtype=torch.float64) * 0.05 + 0.01)
    zeros = torch.randint(0, 2 ** bits, (d_out, d_in // group), generator=g)
    s_x = torch.rand(d_in, generator=g, dtype=torch.float64) * 2 + 0.25
    s_g = torch.rand(d_out, generator=g, dtype=torch.float64) * 2 + 0.25
    return (O.pack_codes(codes, bits), scales.float().numpy(), zeros.numpy().astype(np.uint8),
            s_x.float().numpy(), s_g.float().numpy())


def _run(K, opts, packed, scales, zeros, s_x, s_g, x):
    d_out, d_in = scales.shape[0], x.shape[1]
    desc = torch.empty(K.kronq_matvec_desc_bytes(opts, d_out, d_in), dtype=torch.uint8,
                       device="cuda")
    sx, sg = torch.from_numpy(s_x).cuda(), torch.from_numpy(s_g).cuda()
    K.kronq_matvec_prepare(opts, sx, sg, desc)
    ws = torch.empty(K.kronq_matvec_workspace_bytes(d_out, d_in, x.shape[0]),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty(x.shape[0], d_out, device="cuda")
    info = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    K.kronq_dequant_matvec(opts, desc, torch.from_numpy(packed.view(np.int32)).cuda(),
                           torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(),
                           torch.from_numpy(x).cuda(), y, ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    return y.double().cpu().numpy()


@pytest.mark.parametrize("case", CASES)
def test_dequant_matvec_random_codes(cuda_device, case):
    K = _kq()
    d_out, d_in, rot_out, rot_in, bits, group, nt, flags = case
    packed, scales, zeros, s_x, s_g = _random_layer(d_out, d_in, bits, group, d_out + d_in)
    x = np.random.default_rng(7).standard_normal((nt, d_in)).astype(np.float32)
    opts = K.make_opts(bits=bits, group=group, seed=11, rot_in=rot_in, rot_out=rot_out,
                       flags=flags)
    got = _run(K, opts, packed, scales, zeros, s_x, s_g, x)
    w_hat = O.dequantize(O.unpack_codes(packed, bits, d_in), scales, zeros, group)
    want = O.unrotate_matvec(w_hat, s_x, s_g, x, seed=11, rot_in=rot_in, rot_out=rot_out,
                             no_rot_in=bool(flags & 1), no_rot_out=bool(flags & 2))
    if not flags:
        assert np.array_equal(want, O.dequant_matvec(packed, scales, zeros, bits, group, s_x,
                                                     s_g, x, seed=11, rot_in=rot_in,
                                                     rot_out=rot_out))
    err = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err <= 2e-5, err


def test_dequant_matvec_of_a_quantized_sublayer(cuda_device):
    """Codes from the GPU pipeline itself: the matvec of the quantized layer
    against the oracle's reconstruction from the same codes, and the inputs
    of that matvec (scales, codes, dequantized rows) against the oracle's own
    pipeline (its covariances, BiIP, factor and OBS sweep)."""
    K = _kq()
    from second_order_post_b200.engine import SublayerEngine
    d_out, d_in = 256, 512
    data = synth.small_case(d_out, d_in, 4096, seed=21)
    eng = SublayerEngine(d_out, d_in, bits=4, rot_in=(128, 4), rot_out=(64, 4))
    res = eng.run(data["W"].cuda(), data["X"].cuda(), data["G"].cuda())
    torch.cuda.synchronize()
    eng.check_info()
    x = data["X"][:8].numpy().astype(np.float32)
    packed = res.codes.cpu().numpy().view(np.uint32)
    scales, zeros = res.scales.cpu().numpy(), res.zeros.cpu().numpy()
    s_x, s_g = res.s_x.cpu().numpy(), res.s_g.cpu().numpy()
    got = _run(K, eng.opts, packed, scales, zeros, s_x, s_g, x)
    want = O.dequant_matvec(packed, scales, zeros, 4, 128, s_x, s_g, x, seed=0,
                            rot_in=(128, 4), rot_out=(64, 4))
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 2e-5
    # the oracle's own pipeline
    hx, hg = O.cov(data["X"].numpy()), O.cov(data["G"].numpy())
    wr, hxr, _, sx, sg = O.biip(data["W"].double().numpy(), hx, hg, seed=0,
                                rot_in=(128, 4), rot_out=(64, 4))
    ref = O.obs_quantize(wr, O.chol_inv(hxr, 0.01), 4, 128)
    assert np.allclose(s_x, sx, rtol=1e-5) and np.allclose(s_g, sg, rtol=1e-5)
    eq = O.unpack_codes(packed, 4, d_in) == ref["codes"]
    assert eq.mean() >= 0.999
    # an output row depends on every input row of W only through the output
    # rotation, so a single code resolved the other way at a tie moves all of
    # y; compare where the two pipelines chose the same codes: y of the
    # oracle's rotation applied to the GPU's dequantized rows that agree
    rows = eq.all(axis=1)
    assert rows.mean() >= 0.9
    w_gpu = O.dequantize(O.unpack_codes(packed, 4, d_in), scales, zeros, 128)
    assert np.allclose(w_gpu[rows], ref["w_hat"][rows], rtol=1e-5, atol=1e-7)
