"""kronq_biip_noalloc: BiIP for callers that cannot allocate device memory
(frameworks that own all of HBM through their pool allocator, plugin hosts
that only pass buffers, loops where cudaMalloc would synchronise).

The entry point keeps its scratch in a fixed device array inside the library
instead of a caller workspace. This test calls it through the C ABI twice in
a row, with two different sublayers, and checks each result against the
regular kronq_biip on the same inputs. The second call starts with the first
call's leftovers in the shared array, so a stale-scratch bug would show.

This file is named so that pytest collects it last; it also runs alone.
"""
import pytest
import torch

from second_order_post_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(d_out, d_in, seed, wdtype):
    data = synth.small_case(d_out, d_in, 1024, seed=seed)
    x = data["X"].double()
    g = data["G"].double()
    hx = (x.T @ x / x.shape[0]).float()
    hg = (g.T @ g / g.shape[0]).float()
    return data["W"].to(wdtype), hx, hg


def _run(K, fn, opts, W, hx, hg, ws=None):
    d_out, d_in = W.shape
    Wr = torch.empty(d_out, d_in, device="cuda")
    Hx, Hg = hx.clone().cuda(), hg.clone().cuda()
    sx = torch.empty(d_in, device="cuda")
    sg = torch.empty(d_out, device="cuda")
    info = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    if ws is None:
        fn(opts, W.cuda(), Wr, Hx, Hg, sx, sg, info)
    else:
        fn(opts, W.cuda(), Wr, Hx, Hg, sx, sg, ws, info)
    torch.cuda.synchronize()
    return Wr, Hx, Hg, sx, sg, info.item()


@pytest.mark.parametrize("first,second", [
    ((256, 896, (256, 1), (32, 28), torch.float32),
     (688, 256, (4, 172), (256, 1), torch.bfloat16)),
])
def test_biip_noalloc_matches_biip_twice(cuda_device, first, second):
    from second_order_post_b200 import kronq as K
    for seed, (d_out, d_in, rot_out, rot_in, wdt) in enumerate((first, second)):
        W, hx, hg = _inputs(d_out, d_in, 40 + seed, wdt)
        opts = K.make_opts(seed=5 + seed, rot_in=rot_in, rot_out=rot_out)
        ws = torch.empty(K.kronq_workspace_bytes(K.KRONQ_WS_BIIP, d_out, d_in, opts),
                         dtype=torch.uint8, device="cuda")
        want = _run(K, K.kronq_biip, opts, W, hx, hg, ws)
        got = _run(K, K.kronq_biip_noalloc, opts, W, hx, hg)
        assert want[5] == 0 and got[5] == 0
        # the same kernels on the same inputs, only the scratch lives
        # elsewhere: the results must be bitwise equal (tighter than the 1e-5
        # bar of the BiIP parity tests)
        for g, w in zip(got[:5], want[:5]):
            assert torch.equal(g, w)


def test_biip_noalloc_rejects_bad_sizes(cuda_device):
    from second_order_post_b200 import kronq as K
    W, hx, hg = _inputs(256, 256, 3, torch.float32)
    bad = K.make_opts(rot_in=(128, 3), rot_out=(256, 1))      # 128*3 != 256
    with pytest.raises(K.KronqError) as e:
        _run(K, K.kronq_biip_noalloc, bad, W, hx, hg)
    assert e.value.status == K.KRONQ_ERR_UNSUPPORTED
