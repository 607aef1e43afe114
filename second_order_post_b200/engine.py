"""One-sublayer KronQ quantization on the GPU through libkronq's C ABI.

``SublayerEngine`` owns the device buffers (allocated once with torch, reused
across calls) and enqueues the five steps on one CUDA stream:

  1. kronq_accum_cov(X) -> H_X,  kronq_accum_cov(G) -> H_G
  2. kronq_sensitivity(H_X, H_G)            (before the rotation)
  3. kronq_biip -> W', H_X', H_G', s_x, s_g
  4. kronq_chol_inv(H_X') -> U               (in place)
  5. kronq_quantize_sublayer(W', U) -> codes, scales, zeros, W_hat (in place)

When d_in > d_out, steps 4 and 5 take the split form (kronq_chol_split,
kronq_quantize_split): the same OBS decisions for fewer flops.

All arithmetic runs in the library's kernels; this module only allocates and
passes pointers.
"""
from __future__ import annotations

import dataclasses

import torch

from . import kronq as K


@dataclasses.dataclass
class QuantResult:
    codes: torch.Tensor      # d_out x bits*d_in/32 uint32 words (int32 view)
    scales: torch.Tensor     # d_out x d_in/group fp32
    zeros: torch.Tensor      # d_out x d_in/group uint8
    w_hat: torch.Tensor      # dequantized W' (rotated basis)
    s_x: torch.Tensor
    s_g: torch.Tensor
    sens: torch.Tensor       # float64[3]: tr H_X, tr H_G, product


class SublayerEngine:
    def __init__(self, d_out, d_in, bits=4, group=128, damp_rel=0.01,
                 scale_exp=0.25, seed=0, rot_in=None, rot_out=None, flags=0,
                 device="cuda", keep_w_rot=False, split=None):
        self.d_out, self.d_in = d_out, d_in
        # the split form saves d^3/4 flop in the Cholesky step and spends
        # d_out * (d_in/2)^2 more in the OBS step: worth it when d_in > d_out
        self.split = (d_in > d_out and d_in >= 256) if split is None else split
        self.opts = K.make_opts(bits=bits, group=group, damp_rel=damp_rel,
                                scale_exp=scale_exp, seed=seed,
                                rot_in=rot_in or (d_in, 1),
                                rot_out=rot_out or (d_out, 1), flags=flags)
        dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=dev)
        self.H_X = torch.empty(d_in, d_in, **f32)
        self.H_G = torch.empty(d_out, d_out, **f32)
        self.W_rot = torch.empty(d_out, d_in, **f32)
        self.W_ref = torch.empty(d_out, d_in, **f32) if keep_w_rot else None
        self.s_x = torch.empty(d_in, **f32)
        self.s_g = torch.empty(d_out, **f32)
        self.sens = torch.zeros(3, dtype=torch.float64, device=dev)
        ng = d_in // group
        self.codes = torch.empty(d_out, bits * d_in // 32, dtype=torch.int32, device=dev)
        self.scales = torch.empty(d_out, ng, **f32)
        self.zeros = torch.empty(d_out, ng, dtype=torch.uint8, device=dev)
        # status words: cov X, cov G, BiIP, Cholesky, OBS
        self.info = torch.zeros(5, dtype=torch.int32, device=dev)
        kinds = [K.KRONQ_WS_BIIP, K.KRONQ_WS_CHOL,
                 K.KRONQ_WS_QUANT_SPLIT if self.split else K.KRONQ_WS_QUANT]
        ws = max(K.kronq_workspace_bytes(k, d_out, d_in, self.opts) for k in kinds)
        if ws == 0:
            raise ValueError("unsupported sublayer shape for libkronq")
        self.ws = torch.empty((ws + 255) // 256 * 256, dtype=torch.uint8, device=dev)

    def covariances(self, X, G, stream=None):
        K.kronq_accum_cov(X, self.H_X, 1.0 / X.shape[0], 0.0, self.info[0:1], stream)
        K.kronq_accum_cov(G, self.H_G, 1.0 / G.shape[0], 0.0, self.info[1:2], stream)

    def run(self, W, X, G, stream=None, mark=None, deps=None) -> QuantResult:
        """Enqueue the whole sublayer quantization (no host synchronisation).
        ``mark(name)``, if given, is called after each step is enqueued (the
        benchmark records a CUDA event there). ``deps`` may map "cov_x",
        "cov_g" and "biip" to CUDA events that the stream waits for before X,
        G and W are first read (inputs still arriving on another stream)."""
        mark = mark or (lambda name: None)
        deps = deps or {}
        st = stream or torch.cuda.current_stream()
        if "cov_x" in deps:
            st.wait_event(deps["cov_x"])
        K.kronq_accum_cov(X, self.H_X, 1.0 / X.shape[0], 0.0, self.info[0:1],
                          stream)
        mark("cov_x")
        if "cov_g" in deps:
            st.wait_event(deps["cov_g"])
        K.kronq_accum_cov(G, self.H_G, 1.0 / G.shape[0], 0.0, self.info[1:2],
                          stream)
        mark("cov_g")
        K.kronq_sensitivity(self.H_X, self.H_G, self.sens, stream)
        if "biip" in deps:
            st.wait_event(deps["biip"])
        return self.run_from_covariances(W, stream, mark)

    def run_from_covariances(self, W, stream=None, mark=None, codes=None) -> QuantResult:
        """Steps 3-5 on covariances already in H_X and H_G: BiIP, the damped
        inverse Cholesky factor, OBS with packing. ``codes`` may replace the
        code buffer (a narrower width than the engine was built for)."""
        mark = mark or (lambda name: None)
        codes = self.codes if codes is None else codes
        K.kronq_biip(self.opts, W, self.W_rot, self.H_X, self.H_G, self.s_x,
                     self.s_g, self.ws, self.info[2:3], stream)
        mark("biip")
        if self.W_ref is not None:
            self.W_ref.copy_(self.W_rot)
        if self.split:
            K.kronq_chol_split(self.H_X, self.opts.damp_rel, self.ws,
                               self.info[3:4], stream)
            mark("chol")
            K.kronq_quantize_split(self.opts, self.W_rot, self.H_X, codes,
                                   self.scales, self.zeros, self.ws,
                                   self.info[4:5], stream)
        else:
            K.kronq_chol_inv(self.H_X, self.opts.damp_rel, self.ws, self.info[3:4],
                             stream)
            mark("chol")
            K.kronq_quantize_sublayer(self.opts, self.W_rot, self.H_X, codes,
                                      self.scales, self.zeros, self.ws,
                                      self.info[4:5], stream)
        mark("quant")
        return QuantResult(codes, self.scales, self.zeros, self.W_rot,
                           self.s_x, self.s_g, self.sens)

    def check_info(self):
        """Raises KronqError for a non-zero device status word (syncs)."""
        vals = self.info.tolist()
        names = ("kronq_accum_cov(X)", "kronq_accum_cov(G)", "kronq_biip") + (
            ("kronq_chol_split", "kronq_quantize_split") if self.split else
            ("kronq_chol_inv", "kronq_quantize_sublayer"))
        for name, v in zip(names, vals):
            if v != 0:
                raise K.KronqError(name, v & 0xFF)
