"""A whole model's stack of sublayers: sensitivity scores, greedy bit
allocation, then KronQ quantization of every sublayer at its width
[wmrh §六: mixed precision driven by tr(H_G)·tr(H_X)].

``StackEngine`` keeps every covariance of the stack resident in HBM between
the scoring and the quantization phases (about 2 GB per 7B layer, 64 GB for
32 layers), so each covariance is accumulated once:

  1. per layer: the covariance of each shared input X (q/k/v share one, gate
     and up another) and of each sublayer's output gradients G, then
     kronq_sensitivity per sublayer on the un-rotated covariances;
  2. kronq_allocate_bits over all sublayers' scores and sizes (host);
  3. per sublayer: a working copy of its H_X and its H_G, kronq_biip,
     the damped inverse Cholesky factor and the OBS sweep at its width.

Inputs come from ``synth`` (seeded, generated on the device per layer and
dropped after use). All arithmetic runs in libkronq's kernels.
"""
from __future__ import annotations

import torch

from . import kronq as K
from . import synth
from .engine import SublayerEngine

SCORE_MODES = ("kronq", "trx")   # tr(H_G)·tr(H_X), or tr(H_X) alone


class StackEngine:
    def __init__(self, spec: synth.StackSpec, device="cuda"):
        self.spec = spec
        self.dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=self.dev)
        L, S = spec.layers, len(synth.STACK_SUBLAYERS)
        self.HX = [[torch.empty(d, d, **f32) for _, d in synth.STACK_X_GROUPS]
                   for _ in range(L)]
        self.HG = [[torch.empty(d_out, d_out, **f32)
                    for _, d_out, _, _ in synth.STACK_SUBLAYERS] for _ in range(L)]
        self.sens = torch.zeros(L * S, 3, dtype=torch.float64, device=self.dev)
        self.cov_info = torch.zeros(L, 4 + S, dtype=torch.int32, device=self.dev)
        self._engines = {}
        self.bits = None

    # ------------------------------------------------------------ layout
    @staticmethod
    def n_sublayers(spec) -> int:
        return spec.layers * len(synth.STACK_SUBLAYERS)

    @staticmethod
    def numel(spec):
        return [d_out * d_in for _ in range(spec.layers)
                for _, d_out, d_in, _ in synth.STACK_SUBLAYERS]

    @staticmethod
    def x_group(si: int) -> int:
        g = synth.STACK_SUBLAYERS[si][3]
        return [name for name, _ in synth.STACK_X_GROUPS].index(g)

    def engine(self, d_out, d_in):
        key = (d_out, d_in)
        if key not in self._engines:
            # codes sized for 4 bits; narrower widths use a prefix of the buffer
            self._engines[key] = SublayerEngine(
                d_out, d_in, bits=4, group=self.spec.group, damp_rel=self.spec.damp_rel,
                rot_in=synth.stack_rotation(d_in), rot_out=synth.stack_rotation(d_out),
                device=self.dev, keep_w_rot=True)
        return self._engines[key]

    # ------------------------------------------------------------ phase 1
    def score_layer(self, layer: int, stream=None, timer=None):
        """Covariances of the layer's inputs and gradients, then the
        sensitivity of each sublayer (all on the device)."""
        spec = self.spec
        S = len(synth.STACK_SUBLAYERS)
        info = self.cov_info[layer]
        for gi in range(len(synth.STACK_X_GROUPS)):
            X = synth.make_stack_x(spec, layer, gi, self.dev)
            with _span(timer):
                K.kronq_accum_cov(X, self.HX[layer][gi], 1.0 / X.shape[0], 0.0,
                                  info[gi:gi + 1], stream)
            del X
        for si in range(S):
            G = synth.make_stack_g(spec, layer, si, self.dev)
            with _span(timer):
                K.kronq_accum_cov(G, self.HG[layer][si], 1.0 / G.shape[0], 0.0,
                                  info[4 + si:5 + si], stream)
                K.kronq_sensitivity(self.HX[layer][self.x_group(si)], self.HG[layer][si],
                                    self.sens[layer * S + si], stream)
            del G

    def scores(self, mode="kronq"):
        """Host copies of the scores: tr(H_G)·tr(H_X) ("kronq") or the
        tr(H_X)-only ranking of the ablation ("trx")."""
        if mode not in SCORE_MODES:
            raise ValueError(f"mode must be one of {SCORE_MODES}")
        col = 2 if mode == "kronq" else 0
        return self.sens[:, col].tolist()

    # ------------------------------------------------------------ phase 2
    def allocate(self, mode="kronq"):
        self.bits = K.kronq_allocate_bits(self.scores(mode), self.numel(self.spec),
                                          self.spec.budget)
        return self.bits

    # ------------------------------------------------------------ phase 3
    def quantize_sublayer(self, layer: int, si: int, bits: int, stream=None, timer=None):
        """BiIP, inverse Cholesky factor and OBS of one sublayer at `bits`;
        returns the engine that holds its results (valid until the next call
        on the same shape)."""
        spec = self.spec
        _, d_out, d_in, _ = synth.STACK_SUBLAYERS[si]
        eng = self.engine(d_out, d_in)
        W = synth.make_stack_w(spec, layer, si, self.dev)
        eng.opts.bits = int(bits)
        words = bits * d_in // 32
        eng.codes_view = eng.codes.view(-1)[:d_out * words].view(d_out, words)
        with _span(timer):
            eng.H_X.copy_(self.HX[layer][self.x_group(si)])
            eng.H_G.copy_(self.HG[layer][si])
            eng.run_from_covariances(W, stream, codes=eng.codes_view)
        return eng

    def run(self, mode="kronq", stream=None, timer=None, on_sublayer=None):
        """The whole stack: score, allocate, quantize. ``on_sublayer(layer,
        si, bits, engine)`` sees each sublayer's results."""
        for layer in range(self.spec.layers):
            self.score_layer(layer, stream, timer)
        bits = self.allocate(mode)
        S = len(synth.STACK_SUBLAYERS)
        for layer in range(self.spec.layers):
            for si in range(S):
                eng = self.quantize_sublayer(layer, si, bits[layer * S + si], stream, timer)
                if on_sublayer is not None:
                    on_sublayer(layer, si, bits[layer * S + si], eng)
        return bits

    def check_info(self):
        bad = torch.nonzero(self.cov_info).tolist()
        if bad:
            layer, k = bad[0]
            raise K.KronqError("kronq_accum_cov", int(self.cov_info[layer, k].item()) & 0xFF)
        for eng in self._engines.values():
            eng.check_info()


class _span:
    """Records a pair of CUDA events around a block when a timer list is
    given (device time of the library calls, input generation excluded)."""

    def __init__(self, timer):
        self.timer = timer

    def __enter__(self):
        if self.timer is not None:
            self.e0 = torch.cuda.Event(enable_timing=True)
            self.e0.record()
        return self

    def __exit__(self, *a):
        if self.timer is not None:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record()
            self.timer.append((self.e0, e1))


def device_ms(timer) -> float:
    """Sum of the recorded spans (after a synchronize)."""
    return sum(a.elapsed_time(b) for a, b in timer)


def stack_flops(spec: synth.StackSpec) -> float:
    """Algorithmic flops of one stack pass as executed: each shared input's
    covariance once, n·d(d+1) per covariance, 2d³/3 per Cholesky factor and
    d_out·d_in(d_in-1) per OBS sweep."""
    n = spec.n
    f = 0.0
    for _, d in synth.STACK_X_GROUPS:
        f += n * d * (d + 1)
    for _, d_out, d_in, _ in synth.STACK_SUBLAYERS:
        f += n * d_out * (d_out + 1) + 2 * d_in ** 3 / 3 + d_out * d_in * (d_in - 1)
    return spec.layers * f
