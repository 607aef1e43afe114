"""One sublayer split over ranks (second_order_post_b200.split), run as two
and three gloo ranks on the CPU. The per-rank arithmetic is supplied by the
test (the oracle's steps on this rank's data), so what is checked here is the
product's partition and exchange logic:
  - the token shards' covariances, all-reduced, equal the covariance of all
    tokens (every rank holds the same result);
  - every rank quantizes its own contiguous rows, and the gathered codes,
    scales and zero points equal the single-process sweep in row order.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as O
from second_order_post_b200 import synth
from second_order_post_b200.split import ShardedSublayer, my_rows

D_OUT, D_IN, N, BITS, GROUP = 48, 256, 777, 3, 128
ROT_IN, ROT_OUT, SEED, DAMP = (64, 4), (16, 3), 7, 0.01


class OracleOps:
    """Each rank's local results from the oracle (fp64 on the CPU)."""

    def __init__(self):
        self.H_X = torch.zeros(D_IN, D_IN, dtype=torch.float64)
        self.H_G = torch.zeros(D_OUT, D_OUT, dtype=torch.float64)

    def buffers(self):
        return self.H_X, self.H_G

    def covariance(self, A, H, n_total, slot):
        a = A.double()
        H.copy_(a.T @ a / n_total)

    def sensitivity(self):
        return torch.tensor(O.sensitivity(self.H_X.numpy(), self.H_G.numpy()),
                            dtype=torch.float64)

    def rotate_and_factor(self, W):
        wr, hxr, _, _, _ = O.biip(W.double().numpy(), self.H_X.numpy(), self.H_G.numpy(),
                                  seed=SEED, rot_in=ROT_IN, rot_out=ROT_OUT)
        self.wr, self.u = wr, O.chol_inv(hxr, DAMP)

    def quantize_rows(self, rows):
        res = O.obs_quantize(self.wr[rows.start:rows.stop], self.u, BITS, GROUP)
        codes = O.pack_codes(res["codes"], BITS).view(np.int32)
        return (torch.from_numpy(codes.copy()),
                torch.from_numpy(res["scales"].astype(np.float32)),
                torch.from_numpy(res["zeros"].astype(np.uint8)))


def _data():
    d = synth.small_case(D_OUT, D_IN, N, seed=11)
    return d["W"], d["X"], d["G"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        W, X, G = _data()
        toks = my_rows(N, world, rank)              # this rank's token shard
        sub = ShardedSublayer(D_OUT, D_IN, bits=BITS, group=GROUP, damp_rel=DAMP,
                              seed=SEED, rot_in=ROT_IN, rot_out=ROT_OUT, ops=OracleOps(),
                              device="cpu")
        # the CPU stand-in keeps the covariances in fp64; the collectives
        # run on whatever the buffers are
        res = sub.run(W, X[toks.start:toks.stop], G[toks.start:toks.stop], N)
        torch.save({"codes": res.codes, "scales": res.scales, "zeros": res.zeros,
                    "hx": res.H_X, "hg": res.H_G, "sens": res.sens},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_sublayer_over_gloo_ranks(tmp_path, world):
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    W, X, G = _data()
    # single-process reference: the same steps on all tokens and all rows
    ops = OracleOps()
    ops.covariance(X, ops.H_X, N, 0)
    ops.covariance(G, ops.H_G, N, 1)
    sens = ops.sensitivity()
    ops.rotate_and_factor(W)
    codes, scales, zeros = ops.quantize_rows(range(0, D_OUT))
    for r in range(world):
        got = torch.load(tmp_path / f"rank{r}.pt")
        assert torch.allclose(got["hx"], ops.H_X, rtol=1e-12, atol=1e-15)
        assert torch.allclose(got["hg"], ops.H_G, rtol=1e-12, atol=1e-15)
        assert torch.allclose(got["sens"], sens, rtol=1e-12)
        assert torch.equal(got["codes"], codes)
        assert torch.equal(got["scales"], scales)
        assert torch.equal(got["zeros"], zeros)


@pytest.mark.parametrize("d_out,world", [(48, 2), (48, 5), (7, 3), (2, 4)])
def test_row_shares_partition_the_rows(d_out, world):
    shares = [my_rows(d_out, world, r) for r in range(world)]
    assert [i for s in shares for i in s] == list(range(d_out))
