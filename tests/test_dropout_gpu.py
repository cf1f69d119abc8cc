"""LoRA dropout on the adapter input, on the GPU, against the oracle.

The keep mask is Philox4x32-10 on both sides (written from its published
definition), so the masked input is compared bit for bit; the layer's
outputs and gradients are compared with the fp64 oracle (relative L2 <=
4e-3 and the element-wise bound of tests/common.py), the oracle using the
same keep mask.  Adapter-dominant cases (W = 0, or B of unit variance) put
the masked terms in charge of the whole result.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth
from common import bf16_to_np_f64, bits_f64, check_close, oracle_weight, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,p,seed,offset", [
    (16, 256, 0.05, 1234, 0),
    (37, 640, 0.5, 0xDEADBEEFCAFEF00D, 0x123456789),
    (300, 4096, 0.1, 7, 1 << 40),
    (8, 64, 0.0, 5, 5),
    (64, 128, 0.999, 9, 3),
])
def test_masked_input_bit_exact(M, K, p, seed, offset):
    X = synth.to_bf16_bits(np.random.default_rng(M + K).normal(0, 1, (M, K)).astype(np.float32))
    Xd = to_dev_bf16(X)
    out = q.qlora_dropout_apply(Xd, p, seed, offset).view(torch.int16).cpu().numpy().view(np.uint16)
    keep = oracle.dropout_keep(M, K, p, seed, offset)
    ref = np.where(keep == 1, X, np.uint16(0))
    assert np.array_equal(out, ref)


def run_dropout_case(inp, p, seed, offset, rows=None):
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B, dY = (to_dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    Y = q.qlora_linear_fwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset, U_save=U)
    dX, dA, dB = q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset, dY, U_saved=U)
    dX2, dA2, dB2 = q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset, dY)
    assert q.qlora_device_status() == 0
    # the recompute path forms the same U, so the gradients are identical
    assert torch.equal(dX, dX2) and torch.equal(dA, dA2) and torch.equal(dB, dB2)
    _, _, _, What = oracle_weight(inp["W"])
    Xo, Ao, Bo, dYo = (bits_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    keep = oracle.dropout_keep(M, K, p, seed, offset)
    Yr, Ur = oracle.linear_fwd_dropout(Xo, What, Ao, Bo, alpha, keep, p, rows=rows)
    dXr, dAr, dBr = oracle.linear_bwd_dropout(Xo, What, Ao, Bo, dYo, alpha, keep, p, rows=rows)
    sel = slice(None) if rows is None else rows
    errs = {}
    check_close("Y", bf16_to_np_f64(Y)[sel], Yr, errs)
    check_close("U", bf16_to_np_f64(U)[sel], Ur, errs)
    check_close("dX", bf16_to_np_f64(dX)[sel], dXr, errs)
    check_close("dA", dA.cpu().numpy(), dAr, errs)
    check_close("dB", dB.cpu().numpy(), dBr, errs)
    return errs


@pytest.mark.parametrize("M,N,K,r,p", [
    (1, 512, 256, 8, 0.05),        # a single token (tiled path under dropout)
    (40, 512, 768, 16, 0.3),       # tiled path, split K
    (300, 512, 768, 64, 0.05),     # CTA-pair path
    (257, 384, 640, 24, 0.5),      # ragged M and N, rank not a multiple of 16
])
def test_dropout_layer_against_oracle(M, N, K, r, p):
    run_dropout_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=900 + M), p, seed=42 + M,
                     offset=M * 1000)


@pytest.mark.parametrize("M,N,K,r,p,w_kind", [
    (1, 512, 256, 8, 0.5, "zero"),         # a single token (tiled path under dropout)
    (40, 512, 768, 16, 0.3, "zero"),       # tiled path, split K
    (300, 512, 768, 64, 0.05, "zero"),     # CTA-pair path: dX's masked term is the whole dX
    (257, 384, 640, 24, 0.5, "normal"),    # ragged; B ~ N(0, 1) makes the adapter dominate
])
def test_dropout_adapter_dominant(M, N, K, r, p, w_kind):
    """W = 0 (or B of unit variance): the masked adapter terms are the whole of Y and dX, so
    the masked-add epilogue and the adapter kernel's 1/(1 - p) scales are checked at full
    tolerance rather than under the frozen product's norm."""
    inp = synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1300 + M, weights=w_kind, b_std=1.0)
    run_dropout_case(inp, p, seed=77 + M, offset=M * 31)


@pytest.mark.parametrize("M,N,K,r,p", [(40, 512, 768, 16, 0.3), (300, 512, 768, 64, 0.05)])
def test_kept_dropout_state(M, N, K, r, p):
    """The forward's kept state: Xd_save is bit for bit the masked input and keep_save the
    oracle's keep mask, packed one bit per element; a backward that reads them gives the bits
    of one that generates the mask again."""
    inp = synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1700 + M)
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B, dY = (to_dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    alpha, seed, offset = inp["alpha"], 99 + M, 5 * M
    U = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    Xd = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device="cuda")
    keep = torch.full((M * K // 32,), -1, dtype=torch.int32, device="cuda")
    Y = q.qlora_linear_fwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset, U_save=U, Xd_save=Xd,
                                   keep_save=keep)
    Y0 = q.qlora_linear_fwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset)
    assert torch.equal(Y, Y0)
    assert torch.equal(Xd, q.qlora_dropout_apply(X, p, seed, offset))
    bits = keep.cpu().numpy().view(np.uint32)
    got = ((bits[:, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.uint8).reshape(M, K)
    assert np.array_equal(got, oracle.dropout_keep(M, K, p, seed, offset))
    g_kept = q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset, dY, U_saved=U,
                                        Xd_saved=Xd, keep_saved=keep)
    g_gen = q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, seed, offset, dY, U_saved=U)
    assert q.qlora_device_status() == 0
    for a, b in zip(g_kept, g_gen):
        assert torch.equal(a, b)


def test_dropout_train4096_sampled_rows():
    inp = synth.layer_inputs("train4096")
    rows = np.unique(np.concatenate([np.arange(0, 4096, 131), [0, 4095]]))
    run_dropout_case(inp, 0.05, seed=2024, offset=11, rows=rows)


def test_dropout_p_zero_is_the_plain_layer():
    inp = synth.layer_inputs("tiny", M=70, shape=(512, 512), r=16, seed=3)
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B, dY = (to_dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    U0 = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    U1 = torch.empty_like(U0)
    Y0 = q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, U_save=U0)
    Y1 = q.qlora_linear_fwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, 0.0, 1, 2, U_save=U1)
    assert torch.equal(Y0, Y1) and torch.equal(U0, U1)
    g0 = q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U0)
    g1 = q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, 0.0, 1, 2, dY, U_saved=U1)
    for a, b in zip(g0, g1):
        assert torch.equal(a, b)
