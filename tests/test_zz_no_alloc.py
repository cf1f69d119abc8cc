"""The forward entry point that allocates nothing (qlora_linear_fwd_noalloc).

It serves callers that cannot call cudaMalloc or hand the library a workspace,
for instance a process whose device memory all belongs to another allocator,
or a latency-bound caller that cannot afford cudaMalloc's implicit device
synchronisation.  It runs the same forward as qlora_linear_fwd, with the
library's fixed 4 MiB device scratch in place of the workspace.

Checks, through the C ABI, on each of the three forward paths (few tokens,
the single-CTA tiled GEMM, the CTA-pair GEMM): two calls in a row on different
inputs (the scratch keeps the previous call's contents) give exactly the bits
of qlora_linear_fwd with a caller workspace on Y and U -- the same kernels run
on the same grids, only the scratch's address differs -- and around repeated
calls neither torch's allocator nor the device's free memory moves.  A problem
whose scratch need exceeds 4 MiB is rejected before any launch.  This file is
collected last so that a failure here leaves every other test run.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth
from common import bf16_to_np_f64, to_dev_bf16

pytestmark = pytest.mark.gpu

QLORA_ERR_WORKSPACE = -5


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_call(lib, codes, q8, s2, N, K, X, A, B, alpha, Y, U, M=None):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.qlora_linear_fwd_noalloc(_p(codes), _p(q8), _p(s2), N, K, _p(X), X.shape[0] if M is None else M,
                                        _p(A), _p(B), A.shape[0], float(alpha), _p(Y), _p(U), stream)


CASES = [dict(M=4, shape=(1024, 2048), r=8, seed=40),     # few-token table-lookup path
         dict(M=16, shape=(1024, 2048), r=8, seed=44),    # few-token tensor-memory path, K split over a cluster
         dict(M=100, shape=(768, 1536), r=64, seed=43),    # single-CTA tiled path
         dict(M=300, shape=(512, 768), r=16, seed=41),     # CTA-pair path
         dict(M=1024, shape=(1024, 512), r=64, seed=42)]   # CTA-pair path, several waves


def _case_tensors(c):
    inp = synth.layer_inputs("tiny", M=c["M"], shape=c["shape"], r=c["r"], seed=c["seed"])
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B = (to_dev_bf16(inp[k]) for k in ("X", "A", "B"))
    return inp, codes, q8, s2, X, A, B


def test_noalloc_forward_matches_workspace_forward_twice():
    lib = q.load()
    for c in CASES:
        inp, codes, q8, s2, X, A, B = _case_tensors(c)
        N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
        U_ref = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        Y_ref = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, U_save=U_ref)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        rc = _noalloc_call(lib, codes, q8, s2, N, K, X, A, B, alpha, Y, U)
        assert rc == 0, q.qlora_strerror(rc)
        torch.cuda.synchronize()
        assert q.qlora_device_status() == 0
        assert torch.equal(Y, Y_ref) and torch.equal(U, U_ref), c
        assert np.isfinite(bf16_to_np_f64(Y)).all()


def test_noalloc_forward_allocates_nothing():
    """Repeated calls on every path, after one warm-up call each (the first launch of a kernel
    may load its module): torch's allocated bytes and the device's free bytes are unchanged."""
    lib = q.load()
    prepared = []
    for c in CASES:
        inp, codes, q8, s2, X, A, B = _case_tensors(c)
        N, M, r = inp["N"], inp["M"], inp["r"]
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        args = (lib, codes, q8, s2, N, inp["K"], X, A, B, inp["alpha"], Y, U)
        assert _noalloc_call(*args) == 0
        prepared.append(args)
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        for args in prepared:
            assert _noalloc_call(*args) == 0
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
    assert q.qlora_device_status() == 0


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    lib = q.load()
    inp = synth.layer_inputs("tiny")
    N, K, r, alpha = inp["N"], inp["K"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B = (to_dev_bf16(inp[k]) for k in ("X", "A", "B"))
    Y = torch.empty(inp["M"], N, dtype=torch.bfloat16, device="cuda")
    U = torch.empty(inp["M"], r, dtype=torch.bfloat16, device="cuda")
    # M * r far beyond 4 MiB of scratch: rejected on the host, nothing is launched
    rc = _noalloc_call(lib, codes, q8, s2, N, K, X, A, B, alpha, Y, U, M=1 << 20)
    assert rc == QLORA_ERR_WORKSPACE
    assert q.qlora_device_status() == 0
