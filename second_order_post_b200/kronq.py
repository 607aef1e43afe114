"""Python binding of libkronq.so (include/kronq.h): argument marshalling only.

Every function keeps the C name and argument order; tensors are passed as
device pointers of torch CUDA tensors and the call is enqueued on the current
torch CUDA stream (or ``stream=``). A non-OK status raises ``KronqError``.
There is no fallback: without the compiled library this module raises at
import time.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkronq.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "kronq.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m second_order_post_b200.build` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- constants
KRONQ_OK = 0
KRONQ_ERR_INVALID_ARG = 1
KRONQ_ERR_UNSUPPORTED = 2
KRONQ_ERR_NOT_PD = 3
KRONQ_ERR_NONFINITE = 4
KRONQ_ERR_TIMEOUT = 5
KRONQ_ERR_CUDA = 6
KRONQ_F32 = 0
KRONQ_BF16 = 1
KRONQ_FLAG_NO_ROT_IN = 0x1
KRONQ_FLAG_NO_ROT_OUT = 0x2
KRONQ_FLAG_NO_SCALE = 0x4
KRONQ_WS_BIIP, KRONQ_WS_CHOL, KRONQ_WS_QUANT, KRONQ_WS_LOSS, KRONQ_WS_QUANT_SPLIT = 0, 1, 2, 3, 4


class kronq_rot(ctypes.Structure):
    _fields_ = [("had", ctypes.c_int64), ("m", ctypes.c_int64)]


class kronq_opts(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group", ctypes.c_int32),
                ("block", ctypes.c_int32), ("damp_rel", ctypes.c_float),
                ("scale_exp", ctypes.c_float), ("seed", ctypes.c_uint64),
                ("rot_in", kronq_rot), ("rot_out", kronq_rot),
                ("flags", ctypes.c_uint32)]


def make_opts(bits=4, group=128, block=128, damp_rel=0.01, scale_exp=0.25,
              seed=0, rot_in=(1, 1), rot_out=(1, 1), flags=0) -> kronq_opts:
    return kronq_opts(bits, group, block, damp_rel, scale_exp, seed,
                      kronq_rot(*rot_in), kronq_rot(*rot_out), flags)


class KronqError(RuntimeError):
    def __init__(self, fn, status):
        msg = _lib.kronq_status_string(status).decode()
        if status == KRONQ_ERR_CUDA:
            msg += ": " + _lib.kronq_last_cuda_error().decode()
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_p, _i64, _f, _d, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                         ctypes.c_double, ctypes.c_size_t)
_OPTS = ctypes.POINTER(kronq_opts)
_SIGS = {
    "kronq_accum_cov": [_p, _p, ctypes.c_int, _i64, _i64, _i64, _f, _f, _p, _p],
    "kronq_sensitivity": [_p, _p, _i64, _p, _i64, _p],
    "kronq_biip": [_p, _OPTS, _p, ctypes.c_int, _i64, _i64, _p, _p, _p, _p, _p,
                   _p, _sz, _p],
    "kronq_biip_noalloc": [_p, _OPTS, _p, ctypes.c_int, _i64, _i64, _p, _p, _p,
                           _p, _p, _p],
    "kronq_chol_inv": [_p, _p, _i64, _f, _p, _sz, _p],
    "kronq_quantize_sublayer": [_p, _OPTS, _p, _p, _i64, _i64, _p, _p, _p, _p,
                                _sz, _p],
    "kronq_layer_loss": [_p, _p, _p, _p, _p, _i64, _i64, _p, _p, _sz, _p],
    "kronq_selftest_timeout": [_p, ctypes.c_uint64, _p],
    "kronq_matvec_desc_bytes": [_OPTS, _i64, _i64],
    "kronq_matvec_workspace_bytes": [_i64, _i64, _i64],
    "kronq_matvec_prepare": [_p, _OPTS, _p, _p, _i64, _i64, _p, _sz],
    "kronq_dequant_matvec": [_p, _OPTS, _p, _p, _p, _p, _i64, _i64, _p, _i64, _p, _p, _sz, _p],
    "kronq_chol_split": [_p, _p, _i64, _f, _p, _sz, _p],
    "kronq_chol_split_point": [_i64],
    "kronq_quantize_split": [_p, _OPTS, _p, _p, _i64, _i64, _p, _p, _p, _p, _sz, _p],
    "kronq_gemm_f32": [_p, _i64, _i64, _i64, _f, _p, _i64, ctypes.c_int, _p,
                       _i64, ctypes.c_int, _f, _p, _i64, _p, _sz, _p],
    "kronq_gemm_f32_workspace_bytes": [_i64, _i64, _i64],
    "kronq_workspace_bytes": [ctypes.c_int, _i64, _i64, _OPTS],
    "kronq_allocate_bits": [_p, _p, ctypes.c_int, _d, _p],
    "kronq_status_string": [ctypes.c_int],
    "kronq_kernel_launches": [],
    "kronq_last_cuda_error": [],
}
for _name, _args in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
_lib.kronq_workspace_bytes.restype = ctypes.c_size_t
_lib.kronq_matvec_desc_bytes.restype = ctypes.c_size_t
_lib.kronq_matvec_workspace_bytes.restype = ctypes.c_size_t
_lib.kronq_gemm_f32_workspace_bytes.restype = ctypes.c_size_t
_lib.kronq_chol_split_point.restype = ctypes.c_int64
_lib.kronq_status_string.restype = ctypes.c_char_p
_lib.kronq_kernel_launches.restype = ctypes.c_uint64
_lib.kronq_last_cuda_error.restype = ctypes.c_char_p


def _check(fn, st):
    if st != KRONQ_OK:
        raise KronqError(fn, st)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return KRONQ_BF16
    if t.dtype == torch.float32:
        return KRONQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------- entry points
def kronq_accum_cov(A, H, alpha, beta, info, stream=None):
    """H = alpha * AᵀA + beta * H for A (n x d, bf16/fp32, row-major); info is
    a device int32 word (TIMEOUT when a pipeline wait ran out)."""
    n, d = A.shape
    _check("kronq_accum_cov", _lib.kronq_accum_cov(
        _stream(stream), _ptr(A), _dtype(A), n, d, A.stride(0), alpha, beta,
        _ptr(H), _ptr(info)))


def kronq_sensitivity(H_X, H_G, out, stream=None):
    """out (float64[3], device) = (tr H_X, tr H_G, product)."""
    _check("kronq_sensitivity", _lib.kronq_sensitivity(
        _stream(stream), _ptr(H_X), H_X.shape[0], _ptr(H_G), H_G.shape[0],
        _ptr(out)))


def kronq_workspace_bytes(kind, d_out, d_in, opts=None):
    return int(_lib.kronq_workspace_bytes(
        kind, d_out, d_in, ctypes.byref(opts) if opts is not None else None))


def kronq_biip(opts, W, W_rot, H_X, H_G, s_x, s_g, ws, info, stream=None):
    d_out, d_in = W.shape
    _check("kronq_biip", _lib.kronq_biip(
        _stream(stream), ctypes.byref(opts), _ptr(W), _dtype(W), d_out, d_in,
        _ptr(W_rot), _ptr(H_X), _ptr(H_G), _ptr(s_x), _ptr(s_g), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info)))


def kronq_biip_noalloc(opts, W, W_rot, H_X, H_G, s_x, s_g, info, stream=None):
    """kronq_biip without a workspace, for callers that cannot allocate device
    memory; the library's own fixed device array serves as scratch (calls
    that overlap on the GPU race on it)."""
    d_out, d_in = W.shape
    _check("kronq_biip_noalloc", _lib.kronq_biip_noalloc(
        _stream(stream), ctypes.byref(opts), _ptr(W), _dtype(W), d_out, d_in,
        _ptr(W_rot), _ptr(H_X), _ptr(H_G), _ptr(s_x), _ptr(s_g), _ptr(info)))


def kronq_chol_inv(H, damp_rel, ws, info, stream=None):
    _check("kronq_chol_inv", _lib.kronq_chol_inv(
        _stream(stream), _ptr(H), H.shape[0], damp_rel, _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info)))


def kronq_quantize_sublayer(opts, W_rot, U, codes, scales, zeros, ws, info,
                            stream=None):
    d_out, d_in = W_rot.shape
    _check("kronq_quantize_sublayer", _lib.kronq_quantize_sublayer(
        _stream(stream), ctypes.byref(opts), _ptr(W_rot), _ptr(U), d_out, d_in,
        _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info)))


def kronq_chol_split(H, damp_rel, ws, info, stream=None):
    _check("kronq_chol_split", _lib.kronq_chol_split(
        _stream(stream), _ptr(H), H.shape[0], damp_rel, _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info)))


def kronq_chol_split_point(d):
    return _lib.kronq_chol_split_point(d)


def kronq_quantize_split(opts, W_rot, F, codes, scales, zeros, ws, info,
                         stream=None):
    d_out, d_in = W_rot.shape
    _check("kronq_quantize_split", _lib.kronq_quantize_split(
        _stream(stream), ctypes.byref(opts), _ptr(W_rot), _ptr(F), d_out, d_in,
        _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info)))


def kronq_layer_loss(W_ref, W_hat, H_X, H_G, loss, ws, info, stream=None):
    d_out, d_in = W_ref.shape
    _check("kronq_layer_loss", _lib.kronq_layer_loss(
        _stream(stream), _ptr(W_ref), _ptr(W_hat), _ptr(H_X), _ptr(H_G), d_out,
        d_in, _ptr(loss), _ptr(ws), ws.numel() * ws.element_size(), _ptr(info)))


def kronq_matvec_desc_bytes(opts, d_out, d_in):
    return int(_lib.kronq_matvec_desc_bytes(ctypes.byref(opts), d_out, d_in))


def kronq_matvec_workspace_bytes(d_out, d_in, n_tokens):
    return int(_lib.kronq_matvec_workspace_bytes(d_out, d_in, n_tokens))


def kronq_matvec_prepare(opts, s_x, s_g, desc, stream=None):
    """Fills desc (a uint8 CUDA tensor) with the factors of both sides."""
    _check("kronq_matvec_prepare", _lib.kronq_matvec_prepare(
        _stream(stream), ctypes.byref(opts), _ptr(s_x), _ptr(s_g), s_g.numel(),
        s_x.numel(), _ptr(desc), desc.numel()))


def kronq_dequant_matvec(opts, desc, codes, scales, zeros, x, y, ws, info, stream=None):
    """y (n_tokens x d_out) = the quantized sublayer applied to x (n_tokens x d_in)."""
    n_tokens, d_in = x.shape
    d_out = y.shape[1]
    _check("kronq_dequant_matvec", _lib.kronq_dequant_matvec(
        _stream(stream), ctypes.byref(opts), _ptr(desc), _ptr(codes), _ptr(scales),
        _ptr(zeros), d_out, d_in, _ptr(x), n_tokens, _ptr(y), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info)))


def kronq_selftest_timeout(limit_ns, info, stream=None):
    """Runs the library's bounded device wait on a barrier nothing completes;
    *info becomes KRONQ_ERR_TIMEOUT after about limit_ns (<= 1e9)."""
    _check("kronq_selftest_timeout", _lib.kronq_selftest_timeout(
        _stream(stream), int(limit_ns), _ptr(info)))


def kronq_gemm_f32(A, B, C, info, alpha=1.0, beta=0.0, a_mn=False, b_mn=False,
                   ws=None, stream=None):
    """C = alpha * A Bᵀ + beta * C; A is M x K (or K x M with a_mn), B is
    N x K (or K x N with b_mn); all 2-D fp32 CUDA tensors, rows contiguous.
    ws (a uint8 CUDA tensor) lets large products take the fp16-split path."""
    M, N = C.shape
    K = A.shape[0] if a_mn else A.shape[1]
    _check("kronq_gemm_f32", _lib.kronq_gemm_f32(
        _stream(stream), M, N, K, alpha, _ptr(A), A.stride(0), int(a_mn),
        _ptr(B), B.stride(0), int(b_mn), beta, _ptr(C), C.stride(0),
        None if ws is None else _ptr(ws), 0 if ws is None else ws.numel(),
        _ptr(info)))


def kronq_gemm_f32_workspace_bytes(M, N, K):
    return _lib.kronq_gemm_f32_workspace_bytes(M, N, K)


def kronq_allocate_bits(scores, numel, avg_budget):
    """Host call: greedy 2/3/4-bit allocation (returns a list of ints)."""
    n = len(scores)
    s = (ctypes.c_double * n)(*[float(x) for x in scores])
    m = (ctypes.c_int64 * n)(*[int(x) for x in numel])
    out = (ctypes.c_int * n)()
    _check("kronq_allocate_bits", _lib.kronq_allocate_bits(
        ctypes.cast(s, _p), ctypes.cast(m, _p), n, float(avg_budget),
        ctypes.cast(out, _p)))
    return list(out)


def kronq_status_string(status):
    return _lib.kronq_status_string(status).decode()


def kronq_kernel_launches():
    """Kernels this process has launched through the library so far."""
    return int(_lib.kronq_kernel_launches())


def exported_symbols():
    """Names of the C entry points this binding wraps."""
    return list(_SIGS)
