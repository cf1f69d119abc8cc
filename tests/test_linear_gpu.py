"""Linear layer forward/backward on the GPU against the fp64 oracle.

The oracle quantizes W itself (its codes are independently checked to be
identical to the GPU's), dequantizes to bf16 and evaluates the layer in fp64 on
the exact bf16 operands.  Tolerance: relative L2 <= 4e-3 on every output and
gradient, and beside it an element-wise bound (tests/common.py) so that a few
wrong elements cannot hide in a whole-tensor norm.  Cases span several tiles
with ragged tails in M, N and K, adapter ranks from 8 to 256 (one to four
adapter slices), the tiny and decode workloads in full, and on sampled rows
(dA, dB in full) the 4096^3 training workload, the three weight shapes of the
7B stack and both 65B linears.  Adapter-dominant cases (a zero weight, or B of
unit variance) make the adapter term the whole output on every path, so that
the fused kernels' adapter slices are checked at the same tolerance as the
main product.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth
from common import bf16_to_np_f64, bits_f64, check_close, oracle_weight, oracle_weight_single, to_dev_bf16

pytestmark = pytest.mark.gpu


def run_case(inp, rows=None, check_bwd=True, dy_rows=None, single=False, fp8=False):
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
    Wd = torch.from_numpy(inp["W"]).cuda()
    if single:
        codes, s2 = q.qlora_quantize_nf4(Wd)   # second stage off: s2 = fp32 absmax
        q8 = None
    elif fp8:
        codes, q8, s2 = q.qlora_quantize_nf4_dq_fp8(Wd)
    else:
        codes, q8, s2 = q.qlora_quantize_nf4_dq(Wd)
    X, A, B, dY = (to_dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    Y = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, U_save=U)
    res = {"Y": Y, "U": U}
    if check_bwd:
        dX, dA, dB = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U)
        res.update(dX=dX, dA=dA, dB=dB)
    assert q.qlora_device_status() == 0
    # oracle on the same inputs
    if single:
        What = oracle_weight_single(inp["W"])[2]
    elif fp8:
        rc, rq, rs, _ = oracle.quantize_nf4_dq_fp8(inp["W"].reshape(-1))
        What = bits_f64(oracle.dequant(rc, rq, rs, N * K)[1]).reshape(N, K)
    else:
        What = oracle_weight(inp["W"])[3]
    Xo, Ao, Bo, dYo = (bits_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    Yr, Ur = oracle.linear_fwd(Xo, What, Ao, Bo, alpha, rows=rows)
    sel = slice(None) if rows is None else rows
    errs = {}
    check_close("Y", bf16_to_np_f64(Y)[sel], Yr, errs)
    check_close("U", bf16_to_np_f64(U)[sel], Ur, errs)
    if check_bwd:
        dXr, dAr, dBr = oracle.linear_bwd(Xo, What, Ao, Bo, dYo, alpha, rows=rows)
        check_close("dX", bf16_to_np_f64(res["dX"])[sel], dXr, errs)
        check_close("dA", res["dA"].cpu().numpy(), dAr, errs)
        check_close("dB", res["dB"].cpu().numpy(), dBr, errs)
    return res, errs


def test_tiny_workload_fwd_bwd():
    run_case(synth.layer_inputs("tiny"))


@pytest.mark.parametrize("M,N,K,r", [
    (300, 512, 768, 16),     # ragged M (2 full tiles + 44), several N and K tiles
    (1, 256, 256, 8),        # a single token
    (7, 320, 320, 8),        # ragged N and K tiles (320 = 256 + 64)
    (129, 384, 640, 64),     # one row past a tile; N, K not multiples of 256
    (200, 256, 512, 128),    # two adapter slices
    (64, 512, 256, 256),     # four adapter slices
    (513, 1024, 1152, 24),   # rank not a multiple of 16
])
def test_shapes_and_ranks(M, N, K, r):
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=100 + M))


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_workload_forward(M):
    run_case(synth.layer_inputs("decode", M=M), check_bwd=False)


def test_train4096_sampled_rows():
    inp = synth.layer_inputs("train4096")
    rows = np.unique(np.concatenate([np.arange(0, 4096, 67), [0, 127, 128, 4095]]))
    run_case(inp, rows=rows)


def test_llama7b_down_proj_sampled_rows():
    """The 7B stack's down projection (4096 x 11008, outlier weights), M = 2048."""
    inp = synth.layer_inputs("llama7b", layer=6)
    rows = np.arange(0, 2048, 97)
    run_case(inp, rows=rows)


@pytest.mark.parametrize("layer", [0, 4])
def test_llama7b_attention_and_gate_sampled_rows(layer):
    """The 7B stack's 4096 x 4096 projection and its 11008 x 4096 gate projection (N not a
    multiple of the 512-wide pair tile), outlier weights, M = 2048, at full size in the bench's
    launch configuration: Y, U and dX on sampled rows, dA and dB in full."""
    inp = synth.layer_inputs("llama7b", layer=layer)
    rows = np.unique(np.concatenate([np.arange(0, 2048, 89), [2047]]))
    run_case(inp, rows=rows)


def test_llama65b_square_sampled_rows():
    """The 65B config's 8192 x 8192 linear (Student-t weights), M = 8192, r = 64, at full size:
    Y, U and dX on sampled rows, dA and dB in full."""
    inp = synth.layer_inputs("llama65b", layer=0)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 331), [8191]]))
    run_case(inp, rows=rows)


def test_llama65b_ffn_sampled_rows():
    """The 65B config's 22016 x 8192 linear (Student-t weights), M = 8192, r = 64, at full size
    in the bench's launch configuration: Y, U and dX on 32 sampled rows, dA and dB in full."""
    inp = synth.layer_inputs("llama65b", layer=1)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 263), [8191]]))
    run_case(inp, rows=rows)


def test_gradients_deterministic_and_recompute_path():
    inp = synth.layer_inputs("tiny", M=333, shape=(512, 512), r=32, seed=77)
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B, dY = (to_dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, U_save=U)
    r1 = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U)
    r2 = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U)
    r3 = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=None)
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)
    for a, b in zip(r1, r3):
        assert torch.equal(a, b)
    _, dA4, dB4 = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U, need_dX=False)
    assert torch.equal(dA4, r1[1]) and torch.equal(dB4, r1[2])


def test_zero_adapter_reduces_to_dequant_matmul():
    """B = 0: Y must equal X dequant(W)^T computed by the oracle, adapter grads still flow."""
    inp = synth.layer_inputs("tiny", M=40, shape=(256, 512), r=8, seed=5)
    inp["B"] = np.zeros_like(inp["B"])
    res, errs = run_case(inp)
    assert float(res["dA"].abs().max()) == 0.0


@pytest.mark.parametrize("M,N,K,r,w_kind", [
    (1, 1024, 4096, 8, "zero"),       # table-lookup path
    (4, 4096, 4096, 8, "zero"),       # the decode workload's shape, table-lookup path
    (16, 640, 1024, 64, "zero"),      # tensor-memory few-token path, rank 64
    (16, 1024, 2048, 8, "normal"),    # tensor-memory few-token path, adapter well above the main term
    (40, 512, 768, 16, "zero"),       # tiled path, split K
    (100, 768, 1536, 64, "normal"),   # tiled path
    (300, 512, 768, 64, "zero"),      # CTA-pair path
    (513, 1024, 1152, 24, "normal"),  # CTA-pair path, ragged, rank not a multiple of 16
])
def test_adapter_dominant_layer(M, N, K, r, w_kind):
    """With W = 0 the layer is its adapter alone: Y = s U B^T, dX = s V A, so the adapter
    slices of the fused kernels (forward and dX) carry the whole result.  With B ~ N(0, 1)
    and an ordinary weight the adapter term is several times the main one.  Either way an
    error in the adapter slice cannot shelter under the main product's norm."""
    inp = synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1100 + M, weights=w_kind, b_std=1.0)
    if w_kind == "zero":
        assert not inp["W"].any()
    run_case(inp)


@pytest.mark.parametrize("M,N,K", [(64, 512, 256), (200, 512, 512)])
def test_adapter_slices_filling_every_stage_back_to_back(M, N, K):
    """r = 256 gives as many adapter slices as pipeline stages.  Two calls in a
    row on the same shape with different weights: a stage read before its
    bytes land would return the previous call's data, so the second call
    checks the pipeline's phase handling, not just the arithmetic."""
    for seed in (301, 302):
        run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=256, seed=seed))


@pytest.mark.parametrize("M,N,K,r", [
    (1, 4096, 4096, 8),      # one token (table-lookup kernel)
    (2, 320, 64, 8),         # two tokens, one 64-column block (table-lookup kernel)
    (5, 640, 1024, 24),      # rank not a multiple of 16
    (16, 1024, 640, 64),     # 16 tokens (one 16-token tile), rank 64
    (17, 384, 2048, 16),     # one past a 16-token tile
    (32, 256, 4096, 32),
    (33, 512, 512, 8),       # one past a 32-token tile
    (64, 768, 1536, 64),     # the largest small-M case
])
def test_small_m_forward_and_saved_u(M, N, K, r):
    """Few-token forward: M <= 4 take the table-lookup kernel (tests/test_decode_lut_gpu.py
    has its own cases); 5 <= M <= 32 the tensor-memory kernel, where weight rows and
    adapter rows share the MMA's row side, the K range is split over a cluster and
    U = X A^T is formed per K range in the same launch.  M = 33 and 64 cross into the
    tiled path.  Y and the saved U against the oracle; the backward then uses that saved U."""
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=500 + M))


@pytest.mark.parametrize("M,N,K,r", [
    (1, 4096, 4096, 8),      # few-token path
    (40, 512, 768, 8),       # tiled path, one CTA per tile
    (300, 512, 768, 64),     # CTA-pair path
])
def test_single_quantization_linear(M, N, K, r):
    """The layer on a weight without the second quantization stage (q8 = NULL,
    s2 = fp32 absmax per block): forward and backward against the oracle."""
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=700 + M), single=True)


@pytest.mark.parametrize("M,N,K,r", [
    (1, 4096, 4096, 8),      # few-token path
    (40, 512, 768, 8),       # tiled path
    (300, 512, 768, 64),     # CTA-pair path
])
def test_fp8_second_stage_linear(M, N, K, r):
    """The layer on a weight whose second stage is FP8-E4M3 (sign-tagged s2):
    forward and backward against the oracle."""
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=800 + M), fp8=True)


def test_empty_batch_and_empty_weight():
    """M = 0: the forward writes nothing; the backward's dA and dB are sums over no tokens, so
    both are zero, as the oracle gives (prefilled NaN must be overwritten).  A weight with no
    element quantizes and dequantizes to empty buffers."""
    inp = synth.layer_inputs("tiny")
    N, K, r, alpha = inp["N"], inp["K"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    A, B = to_dev_bf16(inp["A"]), to_dev_bf16(inp["B"])
    X = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    Y = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha)
    assert tuple(Y.shape) == (0, N)
    dA = torch.full((r, K), float("nan"), device="cuda")
    dB = torch.full((N, r), float("nan"), device="cuda")
    dX, dA, dB = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0
    What = oracle_weight(inp["W"])[3]
    _, dAr, dBr = oracle.linear_bwd(np.zeros((0, K)), What, bits_f64(inp["A"]), bits_f64(inp["B"]),
                                    np.zeros((0, N)), alpha)
    assert tuple(dX.shape) == (0, K)
    assert np.array_equal(dA.cpu().numpy(), dAr) and np.array_equal(dB.cpu().numpy(), dBr)
    assert not dAr.any() and not dBr.any()
    # empty weight: no-op quantize and dequantize
    for shape in ((0, 256), (64, 0)):
        c, qq, ss = q.qlora_quantize_nf4_dq(torch.empty(*shape, device="cuda"))
        assert c.numel() == 0 and qq.numel() == 0 and ss.numel() == 0
        assert q.qlora_dequant(c, qq, ss, *shape).numel() == 0
    assert q.qlora_device_status() == 0


def test_caller_workspace_of_any_dtype_and_too_small():
    """A caller workspace is counted in bytes whatever its dtype: a float32 buffer of the
    required size works and gives the same bits as the binding's own; one byte short is
    refused with the workspace error before any launch."""
    inp = synth.layer_inputs("tiny", M=300, shape=(512, 768), r=16, seed=41)
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B = (to_dev_bf16(inp[k]) for k in ("X", "A", "B"))
    need = q.qlora_workspace_bytes(M, N, K, r)
    ws32 = torch.empty((need + 3) // 4, dtype=torch.float32, device="cuda")
    Y0 = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha)
    Y1 = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, workspace=ws32)
    assert torch.equal(Y0, Y1)
    short = torch.empty(need - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QloraError) as e:
        q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, workspace=short)
    assert e.value.code == -5
    assert q.qlora_device_status() == 0


def test_backward_on_two_streams_and_inside_a_graph_capture():
    """The backward forks its gradient kernel to a second stream of the library's.  Two
    backward calls in flight on two streams, and a backward captured in a CUDA graph while an
    uncaptured one runs on another stream, give the bits of a plain call.  The uncaptured
    call must stay out of the capture that holds the second stream."""
    inp = synth.layer_inputs("tiny", M=300, shape=(512, 768), r=16, seed=55)   # CTA-pair path
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B, dY = (to_dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, U_save=U)
    ref = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U)
    torch.cuda.synchronize()

    def bufs():
        out = (torch.full((M, K), float("nan"), dtype=torch.bfloat16, device="cuda"),
               torch.full((r, K), float("nan"), device="cuda"), torch.full((N, r), float("nan"), device="cuda"))
        return out + (torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda"),)

    def bwd(b):
        q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U, dX=b[0], dA=b[1], dB=b[2],
                           workspace=b[3])

    def same(b):
        return all(torch.equal(x, y) for x, y in zip(b[:3], ref))

    s_a, s_b = torch.cuda.Stream(), torch.cuda.Stream()
    b1, b2 = bufs(), bufs()
    torch.cuda.synchronize()
    for s, b in ((s_a, b1), (s_b, b2)):
        with torch.cuda.stream(s):
            bwd(b)
    torch.cuda.synchronize()
    assert same(b1) and same(b2)

    c1, c2 = bufs(), bufs()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s_a, capture_error_mode="relaxed"):
        bwd(c1)                      # captured: the second stream joins this capture
        with torch.cuda.stream(s_b):
            bwd(c2)                  # runs now, outside the capture
    torch.cuda.synchronize()
    assert same(c2)
    assert torch.isnan(c1[1]).all()  # the captured call has not run yet
    g.replay()
    torch.cuda.synchronize()
    assert same(c1)
    del g
    assert q.qlora_device_status() == 0
