"""Host-side checks of libkronq.so that need no GPU: the library loads, every
entry point declared in include/kronq.h is exported, argument validation
rejects bad calls before touching the device, and the host-only calls
(allocator, workspace sizing, status strings) behave."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "second_order_post_b200", "libkronq.so")
HEADER = os.path.join(ROOT, "include", "kronq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kronq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def K():
    if not os.path.exists(LIB):
        from second_order_post_b200 import build
        build.build()
    from second_order_post_b200 import kronq
    return kronq


def test_every_declared_symbol_is_exported(K):
    lib = ctypes.CDLL(LIB)
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(K.exported_symbols())


def test_status_strings(K):
    for s in range(7):
        assert K.kronq_status_string(s) not in ("", "unknown status")
    assert K.kronq_status_string(99) == "unknown status"


def test_last_cuda_error_and_error_text(K):
    """No CUDA call has failed in this process: the diagnostic reads
    "no error", and a KRONQ_ERR_CUDA exception carries the CUDA text."""
    assert K._lib.kronq_last_cuda_error().decode() == "no error"
    e = K.KronqError("kronq_x", K.KRONQ_ERR_CUDA)
    assert str(e).endswith("no error (status 6)")
    assert "no error" not in str(K.KronqError("kronq_x", K.KRONQ_ERR_INVALID_ARG))


def test_invalid_args_rejected_before_device(K):
    lib = K._lib
    nullp = ctypes.c_void_p(0)
    p16 = ctypes.c_void_p(16)
    assert lib.kronq_accum_cov(None, nullp, 0, 8, 8, 8, 1.0, 0.0, nullp, p16) == K.KRONQ_ERR_INVALID_ARG
    assert lib.kronq_accum_cov(None, p16, 7, 8, 8, 8, 1.0, 0.0, p16, p16) == K.KRONQ_ERR_INVALID_ARG
    # the status word is required
    assert lib.kronq_accum_cov(None, p16, 0, 8, 8, 8, 1.0, 0.0, p16, nullp) == K.KRONQ_ERR_INVALID_ARG
    assert lib.kronq_selftest_timeout(None, 0, p16) == K.KRONQ_ERR_INVALID_ARG
    assert lib.kronq_selftest_timeout(None, 2 * 10 ** 9, p16) == K.KRONQ_ERR_INVALID_ARG
    assert lib.kronq_selftest_timeout(None, 1000, nullp) == K.KRONQ_ERR_INVALID_ARG
    assert lib.kronq_sensitivity(None, nullp, 4, nullp, 4, nullp) == K.KRONQ_ERR_INVALID_ARG
    o = K.make_opts(bits=5, rot_in=(256, 1), rot_out=(256, 1))
    p = ctypes.c_void_p(256)
    assert lib.kronq_quantize_sublayer(None, ctypes.byref(o), p, p, 256, 256, p, p,
                                       p, p, 1 << 20, p) == K.KRONQ_ERR_INVALID_ARG
    o = K.make_opts(bits=4, group=100)
    assert lib.kronq_quantize_sublayer(None, ctypes.byref(o), p, p, 256, 256, p, p,
                                       p, p, 1 << 20, p) == K.KRONQ_ERR_UNSUPPORTED
    o = K.make_opts(rot_in=(24, 10), rot_out=(256, 1))      # 24 not a power of 2
    assert lib.kronq_biip(None, ctypes.byref(o), p, 0, 256, 240, p, p, p, p, p, p,
                          1 << 20, p) == K.KRONQ_ERR_UNSUPPORTED
    assert lib.kronq_chol_inv(None, p, 100, 0.01, p, 1 << 20, p) == K.KRONQ_ERR_UNSUPPORTED
    assert lib.kronq_chol_inv(None, p, 128, -1.0, p, 1 << 20, p) == K.KRONQ_ERR_INVALID_ARG
    # gemm: negative sizes, short pitches, misalignment, C overlapping A
    g = lib.kronq_gemm_f32
    q = ctypes.c_void_p(1 << 20)
    assert g(None, -1, 8, 8, 1.0, p, 8, 0, p, 8, 0, 0.0, q, 8, None, 0, p) == \
        K.KRONQ_ERR_INVALID_ARG
    assert g(None, 8, 8, 8, 1.0, p, 4, 0, p, 8, 0, 0.0, q, 8, None, 0, p) == \
        K.KRONQ_ERR_INVALID_ARG
    assert g(None, 8, 8, 8, 1.0, ctypes.c_void_p(260), 8, 0, p, 8, 0, 0.0, q, 8,
             None, 0, p) == K.KRONQ_ERR_UNSUPPORTED
    assert g(None, 8, 8, 8, 1.0, p, 8, 0, q, 8, 0, 0.0, p, 8, None, 0, p) == \
        K.KRONQ_ERR_INVALID_ARG
    assert g(None, 0, 8, 8, 1.0, nullp, 8, 0, nullp, 8, 0, 0.0, nullp, 8, None, 0,
             p) == K.KRONQ_OK
    assert K.kronq_gemm_f32_workspace_bytes(0, 8, 8) == 0
    assert K.kronq_gemm_f32_workspace_bytes(256, 512, 1024) >= 4 * (256 + 512) * 1024


def test_workspace_sizes(K):
    o = K.make_opts(bits=2, rot_in=(1024, 28), rot_out=(8192, 1))
    assert K.kronq_workspace_bytes(K.KRONQ_WS_CHOL, 8192, 28672, o) >= 2 * 14336 * 14336 * 4 // 2
    assert K.kronq_workspace_bytes(K.KRONQ_WS_QUANT, 8192, 28672, o) >= 8192 * 1024 * 4
    assert K.kronq_workspace_bytes(K.KRONQ_WS_BIIP, 8192, 28672, o) > 0
    assert K.kronq_workspace_bytes(K.KRONQ_WS_CHOL, 10, 100, o) == 0


def test_allocator_matches_oracle(K):
    import oracle as O
    rng = np.random.default_rng(0)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        scores = rng.lognormal(0, 2, n)
        if trial % 5 == 0:
            scores[: n // 2] = scores[0]            # ties
        numel = rng.integers(1, 10_000_000, n)
        budget = float(rng.uniform(2.0, 4.2))
        assert K.kronq_allocate_bits(scores, numel, budget) == \
            O.allocate_bits(scores, numel, budget)


def test_allocator_rejects_bad_input(K):
    with pytest.raises(K.KronqError):
        K.kronq_allocate_bits([1.0], [0], 3.0)
    with pytest.raises(K.KronqError):
        K.kronq_allocate_bits([float("nan")], [10], 3.0)
    with pytest.raises(K.KronqError):
        K.kronq_allocate_bits([1.0], [10], 1.5)
