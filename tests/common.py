"""Helpers shared by the tests: device transfers, oracle reference runs, rel-L2 and
element-wise error bounds."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_nf4_quantized_quantize_b200 import synth

# tolerance on floating-point outputs and gradients: relative L2 error against the fp64 oracle
REL_L2_TOL = 4e-3

# Element-wise bound, beside the rel-L2 one:
#     |got - ref| <= ELEM_REL * |ref| + ELEM_ROW * (rms of ref's row).
# The legitimate per-element errors are the bf16 rounding of the output (at most 2^-8 |ref|,
# inside the first term), the bf16 rounding of the adapter operands s U and s V (random: at
# most about 2^-8 / sqrt(3) of the row's rms once summed over the r terms, and as large as the
# output rounding when the adapter dominates the layer) and fp32 accumulation (about 1e-6
# relative).  2^-6 of the row rms is about ten standard deviations of the operand rounding
# where |ref| is near 0, so no correct element fails, while one element at a tile edge that
# is off by a couple of percent of its row's rms does -- an error that a whole-tensor rel-L2
# would absorb.
ELEM_REL = 2.0 ** -7
ELEM_ROW = 2.0 ** -6


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def elem_violations(got, ref) -> np.ndarray:
    """Indices (flat) of the elements of a 2-D result outside the element-wise bound."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    g2 = got.reshape(ref.shape[0], -1) if ref.ndim > 1 else got.reshape(1, -1)
    r2 = ref.reshape(ref.shape[0], -1) if ref.ndim > 1 else ref.reshape(1, -1)
    rms = np.sqrt(np.mean(r2 * r2, axis=1, keepdims=True)) if r2.shape[1] else np.zeros((r2.shape[0], 1))
    bad = ~(np.abs(g2 - r2) <= ELEM_REL * np.abs(r2) + ELEM_ROW * rms)
    return np.flatnonzero(bad)


def check_close(name: str, got, ref, errs: dict | None = None) -> float:
    """Assert rel-L2 <= REL_L2_TOL and the element-wise bound; returns the rel-L2 error."""
    e = rel_l2(got, ref)
    if errs is not None:
        errs[name] = e
    assert e <= REL_L2_TOL, (name, e, errs)
    bad = elem_violations(got, ref)
    if bad.size:
        g = np.asarray(got, np.float64).reshape(-1)
        r = np.asarray(ref, np.float64).reshape(-1)
        i = bad[:4]
        raise AssertionError(f"{name}: {bad.size} elements outside the element-wise bound, "
                             f"first at {i.tolist()}: got {g[i].tolist()} ref {r[i].tolist()}")
    return e


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
