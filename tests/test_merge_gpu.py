"""Adapter merge into the 16-bit base, then re-quantization, on the GPU.

The merged weight bf16(bf16(W) + s B A) is compared bit for bit with the
oracle (same fp64 operation order on both sides, one rounding to bf16), and
the NF4 + double quantization of that merged weight (codes, q8, s2) bit for
bit with the oracle's quantization of the oracle's merged weight.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(N, K, r, seed, b_scale=0.01):
    g = np.random.default_rng(seed)
    W = synth.weight(seed, 0, N, K)
    A = synth.to_bf16_bits(g.normal(0, 1 / np.sqrt(K), (r, K)).astype(np.float32))
    B = synth.to_bf16_bits(g.normal(0, b_scale, (N, r)).astype(np.float32))
    return W, A, B


def _dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("N,K,r,alpha,b_scale", [
    (256, 256, 8, 16.0, 0.01),      # tiny layer
    (333, 192, 24, 16.0, 0.5),      # ragged rows (not a multiple of the 16-row tile), large adapter
    (128, 320, 256, 32.0, 0.05),    # largest rank; K not a multiple of 256
    (4096, 4096, 64, 16.0, 0.01),   # train4096 layer
])
def test_merge_bit_exact_and_requantize(N, K, r, alpha, b_scale):
    W, A, B = _inputs(N, K, r, 40 + r, b_scale)
    ref = oracle.merge_adapter(W, A, B, alpha)
    Wd, Ad, Bd = torch.from_numpy(W).cuda(), _dev_bf16(A), _dev_bf16(B)
    mb = q.qlora_merge_adapter(Wd, Ad, Bd, alpha, dtype=torch.bfloat16)
    mf = q.qlora_merge_adapter(Wd, Ad, Bd, alpha, dtype=torch.float32)
    got = mb.view(torch.int16).cpu().numpy().view(np.uint16)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} merged elements differ, first {bad[:3].tolist()}"
    # the fp32 output holds exactly the same bf16 values
    assert torch.equal(mf, mb.float())
    # re-quantization of the merged 16-bit weight
    codes, q8, s2 = q.qlora_quantize_nf4_dq(mf)
    rf = (ref.astype(np.uint32) << 16).view(np.float32)
    rc, rq, rs, _ = oracle.quantize_nf4_dq(rf.reshape(-1))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(q8.cpu().numpy(), rq)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert q.qlora_device_status() == 0


def test_merge_with_zero_adapter_is_the_bf16_base():
    W, A, _ = _inputs(64, 512, 16, 3)
    B = np.zeros((64, 16), np.uint16)
    m = q.qlora_merge_adapter(torch.from_numpy(W).cuda(), _dev_bf16(A), _dev_bf16(B), 16.0)
    assert torch.equal(m.cpu(), torch.from_numpy(W).to(torch.bfloat16).float())
