"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, builds the same NF4 table as the oracle, and rejects bad
arguments on the host (no GPU is touched: validation precedes any CUDA call).
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return q.load()


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(qlora_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = header_functions()
    assert {"qlora_quantize_nf4_dq", "qlora_dequant", "qlora_linear_fwd", "qlora_linear_bwd"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared <= q.exported_symbols() | declared  # binding covers the header
    assert declared == set(q._binding._SIGNATURES)


def test_checked_build_exports_the_same_symbols(lib):
    """The checked build (QLORA_DEBUG) compiles for sm_100a and exports every declared
    symbol; the ordinary build answers qlora_debug_record with QLORA_ERR_UNAVAILABLE
    without touching a GPU."""
    path = qbuild.build(debug=True)
    assert path.endswith("libqlora_nf4_debug.so") and os.path.exists(path)
    dlib = ctypes.CDLL(path)
    for name in header_functions():
        assert hasattr(dlib, name), name
    out = (ctypes.c_int64 * 4)()
    assert lib.qlora_debug_record(ctypes.byref(out)) == -7
    assert b"checked build" in lib.qlora_strerror(-7)


def test_library_codebook_equals_oracle_bitwise(lib):
    ours = q.qlora_nf4_codebook()
    _, ref = oracle.nf4_codebook()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_strerror(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -99):
        assert isinstance(q.qlora_strerror(code), str) and q.qlora_strerror(code)


def test_workspace_bytes(lib):
    assert q.qlora_workspace_bytes(16, 256, 256, 8) > 0
    assert q.qlora_workspace_bytes(4096, 4096, 4096, 64) > 4096 * 64 * 2
    assert q.qlora_workspace_bytes(0, 256, 256, 8) == 0
    assert q.qlora_workspace_bytes(16, 256, 256, 0) == 0


def _p(v):
    return ctypes.c_void_p(v)


def test_host_validation_without_gpu(lib):
    P = 1 << 20  # a fake, 16-byte-aligned address: validation fails before any use
    null = None
    # quantize: null pointers, bad K
    assert lib.qlora_quantize_nf4_dq(null, 64, 64, _p(P), _p(P), _p(P), null) == -1
    assert lib.qlora_quantize_nf4_dq(_p(P), 64, 63, _p(P), _p(P), _p(P), null) == -2
    assert lib.qlora_quantize_nf4_dq(_p(P + 4), 64, 64, _p(P), _p(P), _p(P), null) == -2
    # dequant: bad dtype
    assert lib.qlora_dequant(_p(P), _p(P), _p(P), 64, 64, _p(P), 7, null) == -1
    args = dict(N=256, K=256, M=16, r=8, alpha=16.0)

    def fwd(codes=P, X=P, M=16, r=8, alpha=16.0, N=256, K=256, Y=P, ws=P, wsb=1 << 30):
        return lib.qlora_linear_fwd(_p(codes) if codes else null, _p(P), _p(P), N, K, _p(X) if X else null, M,
                                    _p(P), _p(P), r, alpha, _p(Y) if Y else null, null, _p(ws) if ws else null,
                                    wsb, null)

    assert fwd(codes=0) == -1
    assert fwd(X=0) == -1
    assert fwd(Y=0) == -1
    assert fwd(K=100) == -2
    assert fwd(N=100) == -2
    assert fwd(M=-1) == -2
    # an empty batch is valid without any buffer or workspace, and touches no device
    assert fwd(M=0, X=0, Y=0, ws=0, wsb=0) == 0
    assert fwd(r=0) == -1
    assert fwd(r=300) == -1
    assert fwd(r=12) == -2
    assert fwd(alpha=float("nan")) == -1
    assert fwd(X=P + 8) == -2
    # everything valid: the first CUDA query fails on a machine without a B200.  (With a GPU
    # visible this call would launch kernels on the fake addresses, so it runs only without one.)
    if not torch.cuda.is_available():
        assert fwd() in (-6, -3)

    def bwd(dY=P, dA=P, dB=P):
        return lib.qlora_linear_bwd(_p(P), _p(P), _p(P), 256, 256, _p(P), 16, _p(P), _p(P), 8, 16.0,
                                    _p(dY) if dY else null, null, null, _p(dA) if dA else null,
                                    _p(dB) if dB else null, _p(P), 1 << 30, null)

    assert bwd(dY=0) == -1
    assert bwd(dA=0) == -1
    assert bwd(dB=0) == -1
    assert bwd(dY=P + 2) == -2
    # an empty weight: the quantizers and the dequantizer are no-ops on NULL buffers
    assert lib.qlora_quantize_nf4_dq(null, 0, 64, null, null, null, null) == 0
    assert lib.qlora_quantize_nf4(null, 64, 0, null, null, null) == 0
    assert lib.qlora_dequant(null, null, null, 0, 64, null, 0, null) == 0
    assert lib.qlora_quantize_nf4_dq(null, -1, 64, null, null, null, null) == -2


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        q.qlora_quantize_nf4_dq(torch.zeros(64, 64))


def test_dropout_host_validation_without_gpu(lib):
    """The dropout entry points refuse p outside [0, 1) (NaN included) and bad shapes before
    touching any device; an empty batch is valid without buffers; the dropout workspace holds
    the plain one plus the masked input and its keep bits."""
    P = 1 << 20
    null = None
    for p in (-0.1, 1.0, 1.5, float("nan")):
        assert lib.qlora_linear_fwd_dropout(_p(P), _p(P), _p(P), 256, 256, _p(P), 16, _p(P), _p(P), 8, 16.0,
                                            p, 1, 0, _p(P), null, null, null, _p(P), 1 << 30, null) == -1
        assert lib.qlora_linear_bwd_dropout(_p(P), _p(P), _p(P), 256, 256, _p(P), 16, _p(P), _p(P), 8, 16.0,
                                            p, 1, 0, _p(P), null, null, null, null, _p(P), _p(P), _p(P), 1 << 30,
                                            null) == -1
    # kept dropout state: the masked input and the keep bits go together, 16-byte aligned
    assert lib.qlora_linear_fwd_dropout(_p(P), _p(P), _p(P), 256, 256, _p(P), 16, _p(P), _p(P), 8, 16.0,
                                        0.1, 1, 0, _p(P), null, _p(P), null, _p(P), 1 << 30, null) == -1
    assert lib.qlora_linear_bwd_dropout(_p(P), _p(P), _p(P), 256, 256, _p(P), 16, _p(P), _p(P), 8, 16.0,
                                        0.1, 1, 0, _p(P), null, null, _p(P), null, _p(P), _p(P), _p(P), 1 << 30,
                                        null) == -1
    assert lib.qlora_linear_fwd_dropout(_p(P), _p(P), _p(P), 256, 256, _p(P), 16, _p(P), _p(P), 8, 16.0,
                                        0.1, 1, 0, _p(P), null, _p(P + 4), _p(P), _p(P), 1 << 30, null) == -2
    for p in (-0.1, 1.0, 1.5, float("nan")):
        assert lib.qlora_dropout_apply(_p(P), 16, 256, p, 1, 0, _p(P), null) == -1
    assert lib.qlora_dropout_apply(_p(P), 16, 100, 0.1, 1, 0, _p(P), null) == -2   # K % 64
    assert lib.qlora_dropout_apply(_p(P), -1, 256, 0.1, 1, 0, _p(P), null) == -2
    assert lib.qlora_dropout_apply(null, 0, 256, 0.1, 1, 0, null, null) == 0       # empty batch
    assert lib.qlora_dropout_apply(null, 16, 256, 0.1, 1, 0, _p(P), null) == -1
    assert lib.qlora_dropout_apply(_p(P + 2), 16, 256, 0.1, 1, 0, _p(P), null) == -2
    M, N, K, r = 4096, 4096, 4096, 64
    plain = q.qlora_workspace_bytes(M, N, K, r)
    assert q.qlora_workspace_bytes_dropout(M, N, K, r) >= plain + M * K * 2 + M * K // 8
    assert q.qlora_workspace_bytes_dropout(0, N, K, r) == 0


def test_merge_host_validation_without_gpu(lib):
    """qlora_merge_adapter refuses a bad output type, r outside [1, 256], a non-finite alpha,
    NULL or unaligned buffers and oversized shapes before touching any device; an empty weight
    is a no-op."""
    P = 1 << 20
    null = None

    def merge(W=P, N=256, K=256, r=8, alpha=16.0, out=P, dtype=1):
        return lib.qlora_merge_adapter(_p(W) if W else null, N, K, _p(P), _p(P), r, alpha,
                                       _p(out) if out else null, dtype, null)

    assert merge(dtype=5) == -1
    assert merge(r=0) == -1 and merge(r=257) == -1
    assert merge(alpha=float("inf")) == -1 and merge(alpha=float("nan")) == -1
    assert merge(W=0) == -1 and merge(out=0) == -1
    assert merge(W=P + 4) == -2
    assert merge(K=100) == -2
    assert merge(N=(1 << 24) + 64) == -2
    assert merge(W=0, N=0, out=0) == 0
