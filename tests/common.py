"""Helpers shared by the tests: device transfers, oracle reference runs, rel-L2."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_nf4_quantized_quantize_b200 import synth

# tolerance on floating-point outputs and gradients: relative L2 error against the fp64 oracle
REL_L2_TOL = 4e-3


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_np_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def bits_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def oracle_weight(W: np.ndarray):
    """Oracle quantize + dequant of an fp32 N x K weight -> (codes, q8, s2, What bf16 as f64 N x K)."""
    N, K = W.shape
    codes, q8, s2, _ = oracle.quantize_nf4_dq(W.reshape(-1))
    _, wb = oracle.dequant(codes, q8, s2, N * K)
    return codes, q8, s2, bits_f64(wb).reshape(N, K)


def oracle_weight_single(W: np.ndarray):
    """Oracle single quantization + dequant -> (codes, absmax, What bf16 as f64 N x K)."""
    N, K = W.shape
    codes, absmax = oracle.quantize_nf4(W.reshape(-1))
    _, wb = oracle.dequant_single(codes, absmax, N * K)
    return codes, absmax, bits_f64(wb).reshape(N, K)
