"""The forward entry point that allocates nothing (qlora_linear_fwd_noalloc).

It serves callers that cannot call cudaMalloc or hand the library a workspace,
for instance a process whose device memory all belongs to another allocator,
or a latency-bound caller that cannot afford cudaMalloc's implicit device
synchronisation.  It runs the same forward as qlora_linear_fwd, with the
library's fixed 4 MiB device scratch in place of the workspace.

Checks, through the C ABI: two calls in a row on different inputs (the
scratch keeps the previous call's contents) each match qlora_linear_fwd with
a caller workspace within the tests' tolerance (rel-L2 <= 4e-3) on Y and U.
A problem whose scratch need exceeds 4 MiB is rejected before any launch.
This file is collected last so that a failure here leaves every other test run.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth
from common import REL_L2_TOL, bf16_to_np_f64, rel_l2, to_dev_bf16

pytestmark = pytest.mark.gpu

QLORA_ERR_WORKSPACE = -5


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_call(lib, codes, q8, s2, N, K, X, A, B, alpha, Y, U, M=None):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.qlora_linear_fwd_noalloc(_p(codes), _p(q8), _p(s2), N, K, _p(X), X.shape[0] if M is None else M,
                                        _p(A), _p(B), A.shape[0], float(alpha), _p(Y), _p(U), stream)


def test_noalloc_forward_matches_workspace_forward_twice():
    lib = q.load()
    cases = [dict(M=300, shape=(512, 768), r=16, seed=41),
             dict(M=1024, shape=(1024, 512), r=64, seed=42)]
    for c in cases:
        inp = synth.layer_inputs("tiny", M=c["M"], shape=c["shape"], r=c["r"], seed=c["seed"])
        N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
        codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
        X, A, B = (to_dev_bf16(inp[k]) for k in ("X", "A", "B"))
        U_ref = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        Y_ref = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, U_save=U_ref)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        rc = _noalloc_call(lib, codes, q8, s2, N, K, X, A, B, alpha, Y, U)
        assert rc == 0, q.qlora_strerror(rc)
        assert q.qlora_device_status() == 0
        assert rel_l2(bf16_to_np_f64(Y), bf16_to_np_f64(Y_ref)) <= REL_L2_TOL
        assert rel_l2(bf16_to_np_f64(U), bf16_to_np_f64(U_ref)) <= REL_L2_TOL
        assert np.isfinite(bf16_to_np_f64(Y)).all()


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
