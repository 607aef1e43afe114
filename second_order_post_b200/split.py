"""One sublayer split across the ranks of a process group (one process per
GPU, NCCL over NVLink).

The steps differ in how they shard [wmrh §二, §四]:

  covariances   the calibration tokens are sharded: each rank accumulates
                its share Σ_r X_rᵀX_r / n into a full d x d buffer and one
                fp32 all-reduce (sum) gives every rank H_X (and H_G). This
                is the dominant work (n·d² flop) and it splits evenly.
  sensitivity   on the reduced covariances, the same on every rank.
  BiIP, U       replicated: every rank rotates W and the covariances and
                factors H_X' itself. The Cholesky recursion does not split
                well over GPUs, and recomputing it costs less wall time than
                factoring on one rank and broadcasting U (the other ranks
                would wait for the factor either way).
  OBS           rows are independent given U [wmrh §四: H_G cancels from the
                column update], so each rank sweeps its contiguous share of
                the d_out rows of W' with the full U and no further
                exchange.
  codes         the packed codes, scales and zero points are all-gathered in
                row order (a sum-reduction of zero-filled buffers, exact for
                integers and for the fp32 scales, since each entry is written
                by exactly one rank).

All arithmetic runs in the ``ops`` object: by default ``LibraryOps``, the
libkronq calls on this rank's GPU. The collectives are torch.distributed
calls on the given group.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from .ranks import my_sublayers


def my_rows(d_out: int, world: int, rank: int) -> range:
    """This rank's contiguous share of the output rows (sizes differ by at
    most one row; the shares partition [0, d_out) in rank order)."""
    return my_sublayers(d_out, world, rank)


@dataclasses.dataclass
class SplitResult:
    codes: torch.Tensor    # d_out x bits*d_in/32 (int32 view of the uint32 words)
    scales: torch.Tensor   # d_out x d_in/group fp32
    zeros: torch.Tensor    # d_out x d_in/group uint8
    sens: torch.Tensor     # float64[3]
    H_X: torch.Tensor      # the reduced covariance (before the rotation)
    H_G: torch.Tensor


class LibraryOps:
    """The per-rank steps as libkronq calls on one GPU (the product path)."""

    def __init__(self, d_out, d_in, bits, group, damp_rel, rot_in, rot_out, seed,
                 device):
        from . import kronq as K
        from .engine import SublayerEngine
        self.K = K
        self.eng = SublayerEngine(d_out, d_in, bits=bits, group=group,
                                  damp_rel=damp_rel, rot_in=rot_in, rot_out=rot_out,
                                  seed=seed, device=device, split=False)
        self.device = self.eng.H_X.device

    def buffers(self):
        return self.eng.H_X, self.eng.H_G

    def covariance(self, A, H, n_total, slot):
        self.K.kronq_accum_cov(A, H, 1.0 / n_total, 0.0, self.eng.info[slot:slot + 1])

    def sensitivity(self):
        self.K.kronq_sensitivity(self.eng.H_X, self.eng.H_G, self.eng.sens)
        return self.eng.sens

    def rotate_and_factor(self, W):
        e = self.eng
        self.K.kronq_biip(e.opts, W, e.W_rot, e.H_X, e.H_G, e.s_x, e.s_g, e.ws,
                          e.info[2:3])
        self.K.kronq_chol_inv(e.H_X, e.opts.damp_rel, e.ws, e.info[3:4])

    def quantize_rows(self, rows: range):
        """OBS of rows [rows.start, rows.stop) of W' with the full U; returns
        (codes, scales, zeros) of those rows."""
        e, K = self.eng, self.K
        r0, r1 = rows.start, rows.stop
        if r1 <= r0:
            return (e.codes[r0:r1], e.scales[r0:r1], e.zeros[r0:r1])
        K.kronq_quantize_sublayer(e.opts, e.W_rot[r0:r1], e.H_X, e.codes[r0:r1],
                                  e.scales[r0:r1], e.zeros[r0:r1], e.ws, e.info[4:5])
        return (e.codes[r0:r1], e.scales[r0:r1], e.zeros[r0:r1])

    def check(self):
        self.eng.check_info()


class ShardedSublayer:
    def __init__(self, d_out, d_in, bits=4, group=128, damp_rel=0.01, seed=0,
                 rot_in=None, rot_out=None, pg=None, ops=None, device="cuda"):
        self.d_out, self.d_in, self.bits, self.group_size = d_out, d_in, bits, group
        self.pg = pg
        self.world = dist.get_world_size(pg)
        self.rank = dist.get_rank(pg)
        self.ops = ops or LibraryOps(d_out, d_in, bits, group, damp_rel,
                                     rot_in or (d_in, 1), rot_out or (d_out, 1), seed,
                                     device)

    def run(self, W, X_local, G_local, n_total: int) -> SplitResult:
        """W: the full weights on every rank; X_local, G_local: this rank's
        token shard; n_total: the tokens over all ranks."""
        ops = self.ops
        H_X, H_G = ops.buffers()
        ops.covariance(X_local, H_X, n_total, 0)
        ops.covariance(G_local, H_G, n_total, 1)
        # the one data-path exchange of the covariances
        dist.all_reduce(H_X, op=dist.ReduceOp.SUM, group=self.pg)
        dist.all_reduce(H_G, op=dist.ReduceOp.SUM, group=self.pg)
        H_X0, H_G0 = H_X.clone(), H_G.clone()
        sens = ops.sensitivity()
        ops.rotate_and_factor(W)
        rows = my_rows(self.d_out, self.world, self.rank)
        codes_l, scales_l, zeros_l = ops.quantize_rows(rows)
        codes, scales, zeros = self._gather_rows(rows, codes_l, scales_l, zeros_l)
        return SplitResult(codes, scales, zeros, sens, H_X0, H_G0)

    def _gather_rows(self, rows, codes_l, scales_l, zeros_l):
        d_out = self.d_out
        dev = codes_l.device
        ng = self.d_in // self.group_size
        words = self.bits * self.d_in // 32
        codes = torch.zeros(d_out, words, dtype=torch.int32, device=dev)
        scales = torch.zeros(d_out, ng, dtype=torch.float32, device=dev)
        zeros = torch.zeros(d_out, ng, dtype=torch.int32, device=dev)
        codes[rows.start:rows.stop] = codes_l
        scales[rows.start:rows.stop] = scales_l
        zeros[rows.start:rows.stop] = zeros_l.to(torch.int32)
        # each entry is written by one rank: the sums are exact
        for t in (codes, scales, zeros):
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.pg)
        return codes, scales, zeros.to(torch.uint8)
