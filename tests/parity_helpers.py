"""Shared parity check for OBS decisions (test infrastructure only)."""
import numpy as np

import oracle as O


def replay_check(w, u, codes, zeros, bits, group, tau=1e-3):
    """Every decision of a candidate must be the oracle's rounding of the
    value it sees given the candidate's own earlier decisions, except within
    tau of a rounding tie. Returns (fraction identical to that decision,
    number of non-tie mismatches, number of tie mismatches)."""
    rep = O.obs_quantize(w, u, bits, group, forced_codes=codes, forced_zeros=zeros)
    maxq = 2 ** bits - 1
    v = rep["v"]
    frac = v - np.floor(v)
    near_tie = np.abs(frac - 0.5) < tau
    near_clamp = (np.abs(v - (maxq + 0.5)) < tau) | (np.abs(v + 0.5) < tau)
    mism = codes != rep["own"]
    bad = mism & ~(near_tie | near_clamp)
    # zero points: rint(-xmin/scale) may differ only at a tie
    zr = rep["zraw"]
    zbad = (zeros != np.rint(zr)) & ~(np.abs(zr - np.floor(zr) - 0.5) < tau)
    return 1.0 - mism.mean(), int(bad.sum()) + int(zbad.sum()), int((mism & ~bad).sum())
