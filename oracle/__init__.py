"""CPU oracle for the QLoRA NF4 + double-quant linear layer.

TEST INFRASTRUCTURE ONLY: the tests, the package's ``smoke()`` check and the
bench's CPU-baseline / reference arm use it; the product library never does.
It shares no code with the CUDA path.

The arithmetic lives in ``nf4_oracle.c`` (plain C, fp64 for the linear layer,
IEEE fp32 with one rounding per operation for the quantizer); this module only
builds that file with gcc and marshals numpy arrays through ctypes.  Each
function cites the passage it follows in the C source:

* codebook: "QLoRAの理論と実装", listing create_nf4_codebook, and §5-1
  "数学的な構成" (8 negative levels, zero, 7 positive levels);
* quantize: same page, §5-1 steps 1-2 and the listing quantize_nf4;
* double quant: same page §5-2, and the Qiita page's "Double Quantization
  の仕組み" (W ~ (c2 * c1_quant) * W_quant);
* dequant: §5-1 step 3 with the two-level constant, to bf16 as the Qiita page's
  storage/compute split requires;
* linear fwd/bwd: "LoRAの復習" (h = W0 x + (alpha/r) B A x), "QLoRAの計算フロー"
  and "逆伝播と勾配の流れ" (dB, dA), dX by the chain rule.

Parity status: every function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_SO = os.path.join(_HERE, "libnf4_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 64
GROUP = 256


def build(force: bool = False) -> str:
    """Compile nf4_oracle.c into libnf4_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_norm_ppf.restype = ctypes.c_double
            lib.oracle_norm_ppf.argtypes = [ctypes.c_double]
            lib.oracle_nf4_codebook.argtypes = [P, P]
            lib.oracle_nearest_code.restype = ctypes.c_int
            lib.oracle_nearest_code.argtypes = [ctypes.c_float, P]
            lib.oracle_quantize_nf4.restype = ctypes.c_int
            lib.oracle_quantize_nf4.argtypes = [P, i64, P, P, P]
            lib.oracle_double_quant.argtypes = [P, i64, P, P]
            lib.oracle_double_quant_fp8.argtypes = [P, i64, P, P]
            lib.oracle_philox4x32_10.argtypes = [P, P, P]
            lib.oracle_dropout_keep.argtypes = [i64, i64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint64, P]
            lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
            lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
            lib.oracle_e4m3_to_f32.restype = ctypes.c_float
            lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
            lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
            lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.oracle_dequant.argtypes = [P, P, P, i64, P, P, P]
            lib.oracle_dequant_single.argtypes = [P, P, i64, P, P, P]
            lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
            lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.oracle_merge_adapter.argtypes = [P, i64, i64, P, P, ctypes.c_int, ctypes.c_double, P]
            lib.oracle_linear_fwd.argtypes = [P, P, P, P, i64, i64, i64, ctypes.c_int,
                                              ctypes.c_double, P, i64, P, P]
            lib.oracle_linear_bwd.argtypes = [P, P, P, P, P, i64, i64, i64, ctypes.c_int,
                                              ctypes.c_double, P, i64, P, P, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_load().oracle_threads())


def norm_ppf(p: float) -> float:
    return float(_load().oracle_norm_ppf(float(p)))


def nf4_codebook():
    """(fp64 levels, fp32 levels) of the NF4 table, ascending."""
    t64 = np.zeros(16, np.float64)
    t32 = np.zeros(16, np.float32)
    _load().oracle_nf4_codebook(_p(t64), _p(t32))
    return t64, t32


def nearest_code(wn: float, table32: np.ndarray | None = None) -> int:
    t = nf4_codebook()[1] if table32 is None else np.ascontiguousarray(table32, np.float32)
    return int(_load().oracle_nearest_code(ctypes.c_float(wn), _p(t)))


def quantize_nf4(w: np.ndarray, table32: np.ndarray | None = None):
    """Blockwise NF4 of a flattened fp32 array -> (packed codes u8[n/2], absmax f32[n/64])."""
    w = np.ascontiguousarray(w, np.float32).reshape(-1)
    t = nf4_codebook()[1] if table32 is None else np.ascontiguousarray(table32, np.float32)
    n = w.size
    if n % BLOCK:
        raise ValueError("element count must be a multiple of 64")
    codes = np.zeros(n // 2, np.uint8)
    absmax = np.zeros(n // BLOCK, np.float32)
    rc = _load().oracle_quantize_nf4(_p(w), n, _p(t), _p(codes), _p(absmax))
    if rc != 0:
        raise ValueError("oracle_quantize_nf4 failed")
    return codes, absmax


def double_quant(absmax: np.ndarray):
    """8-bit re-quantization of absmax in groups of 256 -> (q8 u8[nb], s2 f32[ceil(nb/256)])."""
    a = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    nb = a.size
    q8 = np.zeros(nb, np.uint8)
    s2 = np.zeros((nb + GROUP - 1) // GROUP, np.float32)
    _load().oracle_double_quant(_p(a), nb, _p(q8), _p(s2))
    return q8, s2


def double_quant_fp8(absmax: np.ndarray):
    """FP8-E4M3 re-quantization of absmax in groups of 256 -> (q8 u8[nb], s2 f32 with the sign bit set)."""
    a = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    nb = a.size
    q8 = np.zeros(nb, np.uint8)
    s2 = np.zeros((nb + GROUP - 1) // GROUP, np.float32)
    _load().oracle_double_quant_fp8(_p(a), nb, _p(q8), _p(s2))
    return q8, s2


def f32_to_e4m3(x) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32).reshape(-1)
    f = _load().oracle_f32_to_e4m3
    return np.array([f(float(v)) for v in x], np.uint8)


def e4m3_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, np.uint8).reshape(-1)
    f = _load().oracle_e4m3_to_f32
    return np.array([f(int(v)) for v in b], np.float32)


def quantize_nf4_dq_fp8(w: np.ndarray, table32: np.ndarray | None = None):
    """Two-level quantization with the FP8 second stage -> (codes, q8, s2, absmax)."""
    codes, absmax = quantize_nf4(w, table32)
    q8, s2 = double_quant_fp8(absmax)
    return codes, q8, s2, absmax


def quantize_nf4_dq(w: np.ndarray, table32: np.ndarray | None = None):
    """Full two-level quantization -> (codes, q8, s2, absmax)."""
    codes, absmax = quantize_nf4(w, table32)
    q8, s2 = double_quant(absmax)
    return codes, q8, s2, absmax


def dequant(codes, q8, s2, n: int, table32: np.ndarray | None = None):
    """-> (w32 f32[n], w bf16 bits u16[n])."""
    t = nf4_codebook()[1] if table32 is None else np.ascontiguousarray(table32, np.float32)
    codes = np.ascontiguousarray(codes, np.uint8)
    q8 = np.ascontiguousarray(q8, np.uint8)
    s2 = np.ascontiguousarray(s2, np.float32)
    if codes.size * 2 < n or q8.size * BLOCK < n or s2.size * BLOCK * GROUP < n:
        raise ValueError("buffers too small for n")
    f32 = np.zeros(n, np.float32)
    b16 = np.zeros(n, np.uint16)
    _load().oracle_dequant(_p(codes), _p(q8), _p(s2), n, _p(t), _p(f32), _p(b16))
    return f32, b16


def dequant_single(codes, absmax, n: int, table32: np.ndarray | None = None):
    """Single quantization (no second stage): -> (w32 f32[n], w bf16 bits u16[n])."""
    t = nf4_codebook()[1] if table32 is None else np.ascontiguousarray(table32, np.float32)
    codes = np.ascontiguousarray(codes, np.uint8)
    absmax = np.ascontiguousarray(absmax, np.float32)
    if codes.size * 2 < n or absmax.size * BLOCK < n:
        raise ValueError("buffers too small for n")
    f32 = np.zeros(n, np.float32)
    b16 = np.zeros(n, np.uint16)
    _load().oracle_dequant_single(_p(codes), _p(absmax), n, _p(t), _p(f32), _p(b16))
    return f32, b16


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 to bf16 (nearest, ties to even) in one step with the oracle's C routine."""
    x = np.ascontiguousarray(x, np.float64).reshape(-1)
    f = _load().oracle_f64_to_bf16
    return np.array([f(float(v)) for v in x], np.uint16)


def merge_adapter(W: np.ndarray, A_bits: np.ndarray, B_bits: np.ndarray, alpha: float) -> np.ndarray:
    """bf16 bits of bf16(bf16(W) + s B A) for fp32 W [N, K], bf16-bit A [r, K], B [N, r]."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    A_bits = np.ascontiguousarray(A_bits, np.uint16)
    B_bits = np.ascontiguousarray(B_bits, np.uint16)
    r = A_bits.shape[0]
    if A_bits.shape != (r, K) or B_bits.shape != (N, r):
        raise ValueError("A must be r x K and B N x r")
    out = np.zeros((N, K), np.uint16)
    _load().oracle_merge_adapter(_p(W), N, K, _p(A_bits), _p(B_bits), r, float(alpha), _p(out))
    return out


def philox4x32_10(ctr, key) -> np.ndarray:
    """One Philox4x32-10 block: 4 uint32 outputs for a 4-word counter and 2-word key."""
    c = np.ascontiguousarray(ctr, np.uint32)
    k = np.ascontiguousarray(key, np.uint32)
    out = np.zeros(4, np.uint32)
    _load().oracle_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def dropout_threshold(p: float) -> int:
    """Integer keep threshold floor(p * 2^16) of the fp32 value of p (at most 2^16 - 1 for
    p < 1); an element is kept iff its 16-bit half word >= it."""
    p32 = float(np.float32(p))
    if not 0.0 <= p32 < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return int(np.floor(p32 * 65536.0))


def dropout_keep(M: int, K: int, p: float, seed: int, offset: int) -> np.ndarray:
    """uint8 [M, K] keep mask of the adapter input (1 = kept)."""
    keep = np.zeros((M, K), np.uint8)
    _load().oracle_dropout_keep(M, K, dropout_threshold(p), seed, offset, _p(keep))
    return keep


def dropout_scale(p: float) -> float:
    """1 / (1 - p) of the fp32 value of p, rounded to fp32: the value both sides use."""
    return float(np.float32(1.0 / (1.0 - float(np.float32(p)))))


def linear_fwd_dropout(X, W, A, B, alpha: float, keep, p: float, rows=None):
    """Y = X W^T + s (Xd A^T) B^T and U = Xd A^T with Xd = X * keep / (1 - p), fp64
    (the adapter input of the PEFT LoRA layer goes through dropout, the frozen path does not)."""
    X, W, A, B = (np.asarray(a, np.float64) for a in (X, W, A, B))
    s = alpha / A.shape[0]
    sel = slice(None) if rows is None else rows
    Xd = X[sel] * keep[sel] * dropout_scale(p)
    U = Xd @ A.T
    return X[sel] @ W.T + s * U @ B.T, U


def linear_bwd_dropout(X, W, A, B, dY, alpha: float, keep, p: float, rows=None):
    """dX = dY W + s ((dY B) A) * keep / (1 - p), dA = s (dY B)^T Xd, dB = s dY^T (Xd A^T), fp64."""
    X, W, A, B, dY = (np.asarray(a, np.float64) for a in (X, W, A, B, dY))
    s = alpha / A.shape[0]
    inv = dropout_scale(p)
    Xd = X * keep * inv
    V = dY @ B
    sel = slice(None) if rows is None else rows
    dX = dY[sel] @ W + s * (V[sel] @ A) * keep[sel] * inv
    return dX, s * V.T @ Xd, s * dY.T @ (Xd @ A.T)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) with the oracle's C routine, per element."""
    x = np.ascontiguousarray(x, np.float32).reshape(-1)
    f = _load().oracle_f32_to_bf16
    return np.array([f(float(v)) for v in x], np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64 (bf16 -> fp32 is a 16-bit shift)."""
    b = np.ascontiguousarray(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f64(a):
    return np.ascontiguousarray(a, np.float64)


def linear_fwd(X, W, A, B, alpha: float, rows=None):
    """fp64 Y = X W^T + (alpha/r) (X A^T) B^T; returns (Y, U) (rows only, if given)."""
    X, W, A, B = _f64(X), _f64(W), _f64(A), _f64(B)
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    assert W.shape == (N, K) and A.shape == (r, K) and B.shape == (N, r)
    if rows is None:
        cnt, rp = M, None
    else:
        rows = np.ascontiguousarray(rows, np.int64)
        assert rows.min() >= 0 and rows.max() < M
        cnt, rp = rows.size, _p(rows)
    Y = np.zeros((cnt, N), np.float64)
    U = np.zeros((cnt, r), np.float64)
    _load().oracle_linear_fwd(_p(X), _p(W), _p(A), _p(B), M, N, K, r, float(alpha),
                              rp, cnt if rows is not None else 0, _p(Y), _p(U))
    return Y, U


def linear_bwd(X, W, A, B, dY, alpha: float, rows=None):
    """fp64 (dX, dA, dB); dX only for ``rows`` if given, dA/dB always full."""
    X, W, A, B, dY = _f64(X), _f64(W), _f64(A), _f64(B), _f64(dY)
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    assert dY.shape == (M, N)
    if rows is None:
        cnt, rp = M, None
    else:
        rows = np.ascontiguousarray(rows, np.int64)
        assert rows.min() >= 0 and rows.max() < M
        cnt, rp = rows.size, _p(rows)
    dX = np.zeros((cnt, K), np.float64)
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    _load().oracle_linear_bwd(_p(X), _p(W), _p(A), _p(B), _p(dY), M, N, K, r, float(alpha),
                              rp, cnt if rows is not None else 0, _p(dX), _p(dA), _p(dB))
    return dX, dA, dB
