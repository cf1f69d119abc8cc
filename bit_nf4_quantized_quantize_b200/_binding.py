"""ctypes binding of libqlora_nf4.so with the C ABI's names.

Each function checks tensor dtypes/devices/contiguity, allocates outputs the
caller did not pass (torch device memory), and calls the C entry point with
raw device pointers and torch's current stream.  Non-zero return codes raise
QloraError.

With QLORA_CHECKED_LIBRARY=1 in the environment the binding loads the checked
build, libqlora_nf4_debug.so (bounds and alignment checks before every TMA
copy and cluster exchange; qlora_debug_record reads what they found).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libqlora_nf4_debug.so" if os.environ.get("QLORA_CHECKED_LIBRARY") == "1"
                         else "libqlora_nf4.so")
_lock = threading.Lock()
_lib = None

QLORA_OUT_BF16 = 0
QLORA_OUT_FP32 = 1

_SIGNATURES = {
    "qlora_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_nf4_codebook": (ctypes.c_int, [ctypes.c_void_p]),
    "qlora_quantize_nf4_dq": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_quantize_nf4_dq_fp8": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_quantize_nf4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_merge_adapter": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                           ctypes.c_int, ctypes.c_void_p]),
    "qlora_dequant": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "qlora_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]),
    "qlora_linear_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_linear_bwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "qlora_workspace_bytes_dropout": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]),
    "qlora_linear_fwd_dropout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                                ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear_bwd_dropout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                                ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_dropout_apply": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float,
                                           ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_selftest_device_timeout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_timing_enable": (ctypes.c_int, [ctypes.c_int]),
    "qlora_timing_collect": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]),
    "qlora_launch_count": (ctypes.c_int64, []),
    "qlora_debug_record": (ctypes.c_int, [ctypes.c_void_p]),
}

KERNEL_KINDS = ["quantize", "dequant", "lora_gemm", "lora_reduce", "fwd_fused", "dx_fused", "grad_gemm",
                "grad_reduce", "fwd_decode", "merge", "dropout"]


class QloraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {qlora_strerror(code)} (code {code})")


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libqlora_nf4.so (raises if it was not built: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: run __graft_entry__.build() "
                                   "(python -m bit_nf4_quantized_quantize_b200.build)")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def exported_symbols():
    lib = load()
    return {n for n in _SIGNATURES if hasattr(lib, n)}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device.index != torch.cuda.current_device():
        raise ValueError(f"stream is on {stream.device}; the library launches on the current device "
                         f"cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise QloraError(rc, where)


def _dev(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}; the library launches on the current device "
                         f"cuda:{torch.cuda.current_device()} (use torch.cuda.device)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def qlora_strerror(code: int) -> str:
    return load().qlora_strerror(int(code)).decode()


def qlora_nf4_codebook():
    """The 16 NF4 levels (fp32, ascending) the library quantizes against (host call)."""
    import numpy as np
    out = np.zeros(16, np.float32)
    _check(load().qlora_nf4_codebook(out.ctypes.data_as(ctypes.c_void_p)), "qlora_nf4_codebook")
    return out


def quant_sizes(n_out: int, k_in: int):
    n = n_out * k_in
    nb = n // 64
    return n // 2, nb, (nb + 255) // 256


def qlora_quantize_nf4_dq(W, codes=None, q8=None, s2=None, stream=None):
    """NF4 + double quantization of a fp32 [N, K] CUDA tensor -> (codes, q8, s2)."""
    _dev(W, torch.float32, "W")
    if W.dim() != 2:
        raise ValueError("W must be 2-D [n_out, k_in]")
    N, K = W.shape
    nc, nb, ng = quant_sizes(N, K)
    dev = W.device
    codes = torch.empty(nc, dtype=torch.uint8, device=dev) if codes is None else _dev(codes, torch.uint8, "codes", (nc,))
    q8 = torch.empty(nb, dtype=torch.uint8, device=dev) if q8 is None else _dev(q8, torch.uint8, "q8", (nb,))
    s2 = torch.empty(ng, dtype=torch.float32, device=dev) if s2 is None else _dev(s2, torch.float32, "s2", (ng,))
    _check(load().qlora_quantize_nf4_dq(_ptr(W), N, K, _ptr(codes), _ptr(q8), _ptr(s2), _stream(stream)),
           "qlora_quantize_nf4_dq")
    return codes, q8, s2


def qlora_quantize_nf4_dq_fp8(W, codes=None, q8=None, s2=None, stream=None):
    """NF4 + double quantization with the FP8-E4M3 second stage -> (codes, q8, s2);
    s2 carries its sign bit set, which every consumer reads as the FP8 format."""
    _dev(W, torch.float32, "W")
    if W.dim() != 2:
        raise ValueError("W must be 2-D [n_out, k_in]")
    N, K = W.shape
    nc, nb, ng = quant_sizes(N, K)
    dev = W.device
    codes = torch.empty(nc, dtype=torch.uint8, device=dev) if codes is None else _dev(codes, torch.uint8, "codes", (nc,))
    q8 = torch.empty(nb, dtype=torch.uint8, device=dev) if q8 is None else _dev(q8, torch.uint8, "q8", (nb,))
    s2 = torch.empty(ng, dtype=torch.float32, device=dev) if s2 is None else _dev(s2, torch.float32, "s2", (ng,))
    _check(load().qlora_quantize_nf4_dq_fp8(_ptr(W), N, K, _ptr(codes), _ptr(q8), _ptr(s2), _stream(stream)),
           "qlora_quantize_nf4_dq_fp8")
    return codes, q8, s2


def _weight(codes, q8, s2, n_out: int, k_in: int):
    """Check a quantized weight: (codes, q8, s2) with double quantization, or
    (codes, None, absmax) with single quantization (s2 = fp32 absmax per block)."""
    nc, nb, ng = quant_sizes(n_out, k_in)
    _dev(codes, torch.uint8, "codes", (nc,))
    if q8 is None:
        _dev(s2, torch.float32, "absmax", (nb,))
    else:
        _dev(q8, torch.uint8, "q8", (nb,))
        _dev(s2, torch.float32, "s2", (ng,))


def qlora_quantize_nf4(W, codes=None, absmax=None, stream=None):
    """NF4 without the second stage (single quantization) of a fp32 [N, K] CUDA
    tensor -> (codes, absmax); use (codes, None, absmax) as the weight."""
    _dev(W, torch.float32, "W")
    if W.dim() != 2:
        raise ValueError("W must be 2-D [n_out, k_in]")
    N, K = W.shape
    nc, nb, _ = quant_sizes(N, K)
    dev = W.device
    codes = torch.empty(nc, dtype=torch.uint8, device=dev) if codes is None else _dev(codes, torch.uint8, "codes", (nc,))
    absmax = torch.empty(nb, dtype=torch.float32, device=dev) if absmax is None else _dev(absmax, torch.float32, "absmax", (nb,))
    _check(load().qlora_quantize_nf4(_ptr(W), N, K, _ptr(codes), _ptr(absmax), _stream(stream)), "qlora_quantize_nf4")
    return codes, absmax


def qlora_dequant(codes, q8, s2, n_out: int, k_in: int, out=None, dtype=torch.bfloat16, stream=None):
    """Dense [N, K] dequantized weight (bf16 or fp32)."""
    _weight(codes, q8, s2, n_out, k_in)
    if dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("dtype must be bfloat16 or float32")
    if out is None:
        out = torch.empty(n_out, k_in, dtype=dtype, device=codes.device)
    else:
        _dev(out, dtype, "out", (n_out, k_in))
    code = QLORA_OUT_BF16 if dtype == torch.bfloat16 else QLORA_OUT_FP32
    _check(load().qlora_dequant(_ptr(codes), _ptr(q8), _ptr(s2), n_out, k_in, _ptr(out), code, _stream(stream)),
           "qlora_dequant")
    return out


def qlora_merge_adapter(W, A, B, alpha: float, out=None, dtype=torch.float32, stream=None):
    """Merged 16-bit weight bf16(bf16(W) + (alpha/r) B A) of the fp32 base W [N, K] and the
    adapter A [r, K], B [N, r] (bf16); fp32 output (bf16 values) feeds re-quantization."""
    _dev(W, torch.float32, "W")
    if W.dim() != 2:
        raise ValueError("W must be 2-D [n_out, k_in]")
    N, K = W.shape
    r = A.shape[0]
    _dev(A, torch.bfloat16, "A", (r, K))
    _dev(B, torch.bfloat16, "B", (N, r))
    if dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("dtype must be bfloat16 or float32")
    out = torch.empty(N, K, dtype=dtype, device=W.device) if out is None else _dev(out, dtype, "out", (N, K))
    code = QLORA_OUT_BF16 if dtype == torch.bfloat16 else QLORA_OUT_FP32
    _check(load().qlora_merge_adapter(_ptr(W), N, K, _ptr(A), _ptr(B), r, float(alpha), _ptr(out), code,
                                      _stream(stream)), "qlora_merge_adapter")
    return out


def qlora_workspace_bytes(M: int, n_out: int, k_in: int, r: int) -> int:
    return int(load().qlora_workspace_bytes(M, n_out, k_in, r))


def _nbytes(ws):
    return 0 if ws is None else ws.numel() * ws.element_size()


def _workspace(ws, M, N, K, r, device):
    if M == 0:
        return ws   # an empty batch needs no workspace
    need = qlora_workspace_bytes(M, N, K, r)
    if need == 0:
        raise QloraError(-2, "qlora_workspace_bytes")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    else:
        _dev(ws, ws.dtype, "workspace")
    return ws


def qlora_linear_fwd(codes, q8, s2, n_out: int, k_in: int, X, A, B, alpha: float,
                     Y=None, U_save=None, workspace=None, stream=None):
    """Y = X dequant(W)^T + (alpha/r) (X A^T) B^T in bf16; returns Y (and fills U_save if given)."""
    _weight(codes, q8, s2, n_out, k_in)
    M = X.shape[0]
    r = A.shape[0]
    _dev(X, torch.bfloat16, "X", (M, k_in))
    _dev(A, torch.bfloat16, "A", (r, k_in))
    _dev(B, torch.bfloat16, "B", (n_out, r))
    Y = torch.empty(M, n_out, dtype=torch.bfloat16, device=X.device) if Y is None else _dev(Y, torch.bfloat16, "Y", (M, n_out))
    if U_save is not None:
        _dev(U_save, torch.bfloat16, "U_save", (M, r))
    ws = _workspace(workspace, M, n_out, k_in, r, X.device)
    _check(load().qlora_linear_fwd(_ptr(codes), _ptr(q8), _ptr(s2), n_out, k_in, _ptr(X), M, _ptr(A), _ptr(B), r,
                                   float(alpha), _ptr(Y), _ptr(U_save), _ptr(ws), _nbytes(ws), _stream(stream)),
           "qlora_linear_fwd")
    return Y


def qlora_linear_fwd_noalloc(codes, q8, s2, n_out: int, k_in: int, X, A, B, alpha: float,
                             Y=None, U_save=None, stream=None):
    """qlora_linear_fwd using the library's fixed 4 MiB device scratch (no workspace, no allocation
    inside the library; the binding still allocates Y here if the caller passes none)."""
    _weight(codes, q8, s2, n_out, k_in)
    M = X.shape[0]
    r = A.shape[0]
    _dev(X, torch.bfloat16, "X", (M, k_in))
    _dev(A, torch.bfloat16, "A", (r, k_in))
    _dev(B, torch.bfloat16, "B", (n_out, r))
    Y = torch.empty(M, n_out, dtype=torch.bfloat16, device=X.device) if Y is None else _dev(Y, torch.bfloat16, "Y", (M, n_out))
    if U_save is not None:
        _dev(U_save, torch.bfloat16, "U_save", (M, r))
    _check(load().qlora_linear_fwd_noalloc(_ptr(codes), _ptr(q8), _ptr(s2), n_out, k_in, _ptr(X), M, _ptr(A),
                                           _ptr(B), r, float(alpha), _ptr(Y), _ptr(U_save), _stream(stream)),
           "qlora_linear_fwd_noalloc")
    return Y


def qlora_linear_bwd(codes, q8, s2, n_out: int, k_in: int, X, A, B, alpha: float, dY, U_saved=None,
                     dX=None, dA=None, dB=None, need_dX=True, workspace=None, stream=None):
    """(dX bf16 [M,K] or None, dA fp32 [r,K], dB fp32 [N,r])."""
    _weight(codes, q8, s2, n_out, k_in)
    M = X.shape[0]
    r = A.shape[0]
    _dev(X, torch.bfloat16, "X", (M, k_in))
    _dev(A, torch.bfloat16, "A", (r, k_in))
    _dev(B, torch.bfloat16, "B", (n_out, r))
    _dev(dY, torch.bfloat16, "dY", (M, n_out))
    if U_saved is not None:
        _dev(U_saved, torch.bfloat16, "U_saved", (M, r))
    dev = X.device
    if need_dX:
        dX = torch.empty(M, k_in, dtype=torch.bfloat16, device=dev) if dX is None else _dev(dX, torch.bfloat16, "dX", (M, k_in))
    else:
        dX = None
    dA = torch.empty(r, k_in, dtype=torch.float32, device=dev) if dA is None else _dev(dA, torch.float32, "dA", (r, k_in))
    dB = torch.empty(n_out, r, dtype=torch.float32, device=dev) if dB is None else _dev(dB, torch.float32, "dB", (n_out, r))
    ws = _workspace(workspace, M, n_out, k_in, r, dev)
    _check(load().qlora_linear_bwd(_ptr(codes), _ptr(q8), _ptr(s2), n_out, k_in, _ptr(X), M, _ptr(A), _ptr(B), r,
                                   float(alpha), _ptr(dY), _ptr(U_saved), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                                   _nbytes(ws), _stream(stream)),
           "qlora_linear_bwd")
    return dX, dA, dB


def qlora_workspace_bytes_dropout(M: int, n_out: int, k_in: int, r: int) -> int:
    return int(load().qlora_workspace_bytes_dropout(M, n_out, k_in, r))


def _workspace_dropout(ws, M, N, K, r, device):
    if M == 0:
        return ws   # an empty batch needs no workspace
    need = qlora_workspace_bytes_dropout(M, N, K, r)
    if need == 0:
        raise QloraError(-2, "qlora_workspace_bytes_dropout")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    else:
        _dev(ws, ws.dtype, "workspace")
    return ws


def _dropout_state(Xd, keep, M: int, k_in: int, names):
    """Validate kept dropout state: bf16 [M, K] masked input and int32 [M*K/32] keep words, both or neither."""
    if (Xd is None) != (keep is None):
        raise ValueError(f"{names[0]} and {names[1]} go together")
    if Xd is not None:
        _dev(Xd, torch.bfloat16, names[0], (M, k_in))
        _dev(keep, torch.int32, names[1], (M * k_in // 32,))


def qlora_linear_fwd_dropout(codes, q8, s2, n_out: int, k_in: int, X, A, B, alpha: float, p: float, seed: int,
                             offset: int, Y=None, U_save=None, Xd_save=None, keep_save=None, workspace=None,
                             stream=None):
    """The forward with dropout p on the adapter input (Philox keep mask from seed, offset).
    Xd_save (bf16 [M, K]) and keep_save (int32 [M*K/32]), if given, receive the masked input
    and the keep bits, for the backward to read instead of generating the mask again."""
    _weight(codes, q8, s2, n_out, k_in)
    M = X.shape[0]
    r = A.shape[0]
    _dev(X, torch.bfloat16, "X", (M, k_in))
    _dev(A, torch.bfloat16, "A", (r, k_in))
    _dev(B, torch.bfloat16, "B", (n_out, r))
    Y = torch.empty(M, n_out, dtype=torch.bfloat16, device=X.device) if Y is None else _dev(Y, torch.bfloat16, "Y", (M, n_out))
    if U_save is not None:
        _dev(U_save, torch.bfloat16, "U_save", (M, r))
    _dropout_state(Xd_save, keep_save, M, k_in, ("Xd_save", "keep_save"))
    ws = _workspace_dropout(workspace, M, n_out, k_in, r, X.device)
    _check(load().qlora_linear_fwd_dropout(_ptr(codes), _ptr(q8), _ptr(s2), n_out, k_in, _ptr(X), M, _ptr(A),
                                           _ptr(B), r, float(alpha), float(p), int(seed), int(offset), _ptr(Y),
                                           _ptr(U_save), _ptr(Xd_save), _ptr(keep_save), _ptr(ws), _nbytes(ws),
                                           _stream(stream)),
           "qlora_linear_fwd_dropout")
    return Y


def qlora_linear_bwd_dropout(codes, q8, s2, n_out: int, k_in: int, X, A, B, alpha: float, p: float, seed: int,
                             offset: int, dY, U_saved=None, dX=None, dA=None, dB=None, need_dX=True,
                             Xd_saved=None, keep_saved=None, workspace=None, stream=None):
    """The backward with dropout p on the adapter input -> (dX or None, dA, dB).  Xd_saved and
    keep_saved: the state a forward kept (same p, seed, offset), or None to generate the mask."""
    _weight(codes, q8, s2, n_out, k_in)
    M = X.shape[0]
    r = A.shape[0]
    _dev(X, torch.bfloat16, "X", (M, k_in))
    _dev(A, torch.bfloat16, "A", (r, k_in))
    _dev(B, torch.bfloat16, "B", (n_out, r))
    _dev(dY, torch.bfloat16, "dY", (M, n_out))
    if U_saved is not None:
        _dev(U_saved, torch.bfloat16, "U_saved", (M, r))
    dev = X.device
    if need_dX:
        dX = torch.empty(M, k_in, dtype=torch.bfloat16, device=dev) if dX is None else _dev(dX, torch.bfloat16, "dX", (M, k_in))
    else:
        dX = None
    dA = torch.empty(r, k_in, dtype=torch.float32, device=dev) if dA is None else _dev(dA, torch.float32, "dA", (r, k_in))
    dB = torch.empty(n_out, r, dtype=torch.float32, device=dev) if dB is None else _dev(dB, torch.float32, "dB", (n_out, r))
    _dropout_state(Xd_saved, keep_saved, M, k_in, ("Xd_saved", "keep_saved"))
    ws = _workspace_dropout(workspace, M, n_out, k_in, r, dev)
    _check(load().qlora_linear_bwd_dropout(_ptr(codes), _ptr(q8), _ptr(s2), n_out, k_in, _ptr(X), M, _ptr(A),
                                           _ptr(B), r, float(alpha), float(p), int(seed), int(offset), _ptr(dY),
                                           _ptr(U_saved), _ptr(Xd_saved), _ptr(keep_saved), _ptr(dX), _ptr(dA),
                                           _ptr(dB), _ptr(ws), _nbytes(ws), _stream(stream)),
           "qlora_linear_bwd_dropout")
    return dX, dA, dB


def qlora_dropout_apply(X, p: float, seed: int, offset: int, out=None, stream=None):
    """X * keep (bf16, dropped elements 0): the masked adapter input of the dropout calls."""
    M, K = X.shape
    _dev(X, torch.bfloat16, "X", (M, K))
    out = torch.empty_like(X) if out is None else _dev(out, torch.bfloat16, "out", (M, K))
    _check(load().qlora_dropout_apply(_ptr(X), M, K, float(p), int(seed), int(offset), _ptr(out), _stream(stream)),
           "qlora_dropout_apply")
    return out


def qlora_device_status(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error flag as a QLORA_* code."""
    return int(load().qlora_device_status(_stream(stream)))


def qlora_timing_enable(on: bool = True) -> None:
    _check(load().qlora_timing_enable(1 if on else 0), "qlora_timing_enable")


def qlora_timing_collect() -> dict:
    """{kind: (total_ms, launches)} of the kernels launched since timing was enabled."""
    import numpy as np
    ms = np.zeros(len(KERNEL_KINDS), np.float64)
    cnt = np.zeros(len(KERNEL_KINDS), np.int64)
    _check(load().qlora_timing_collect(ms.ctypes.data_as(ctypes.c_void_p), cnt.ctypes.data_as(ctypes.c_void_p),
                                       len(KERNEL_KINDS)), "qlora_timing_collect")
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS) if cnt[i]}


def qlora_debug_record() -> dict:
    """Read and clear the checked build's record of failed checks (current device):
    {failed, first_code, first_value, first_cta}.  The ordinary build raises QloraError."""
    out = (ctypes.c_int64 * 4)()
    _check(load().qlora_debug_record(ctypes.byref(out)), "qlora_debug_record")
    return {"failed": int(out[0]), "first_code": int(out[1]), "first_value": int(out[2]), "first_cta": int(out[3])}


def qlora_launch_count() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(load().qlora_launch_count())


def qlora_selftest_device_timeout(waited_ns=None, stream=None):
    """Enqueue the library's expired-wait diagnostic (see include/qlora_nf4.h)."""
    if waited_ns is not None:
        _dev(waited_ns, torch.int64, "waited_ns", (1,))
    _check(load().qlora_selftest_device_timeout(_ptr(waited_ns), _stream(stream)), "qlora_selftest_device_timeout")
