"""Seeded synthetic inputs for the QLoRA NF4 linear layer.

This module only draws random numbers; it holds none of the method's
arithmetic.  The CUDA path, the CPU oracle, the tests and the bench all take
their inputs from here, so that both sides of every comparison see the same
bytes.

Every stream is numpy's Philox4x32-10 generator (Salmon et al., SC'11) keyed by
(workload seed, tensor id).  Normals come from numpy's generator; bf16 tensors
are fp32 draws rounded to nearest-even bf16 (returned as uint16 bit patterns).

Workloads (weights are N x K = out x in, activations are M tokens x K):

* ``tiny``       256x256, M=16, r=8, alpha=16 (A ~ N(0, 1/256), B ~ N(0, 0.01^2)).
* ``decode``     4096x4096, M in {1, 4, 16}, r=8, alpha=16, forward only.
* ``train4096``  4096x4096, M=4096, r=64, alpha=16, forward + backward.
* ``llama7b``    q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008, M=2048,
                 r=64; weights N(0, 0.02^2) with 0.1% of entries set to +-6 sigma.
* ``llama65b``   8192x8192 and 22016x8192, M=8192, r=64; weights Student-t
                 (nu=4) scaled to std 0.02.

W ~ N(0, 0.02^2) unless stated; X, dY ~ N(0, 1); A ~ N(0, 1/K); B ~ N(0, 0.01^2).
Test cases may override the weight kind (``zero``: an all-zero weight) and B's
standard deviation, to make the adapter term dominate the layer.
"""
from __future__ import annotations

import numpy as np

WEIGHT_STD = 0.02

# tensor ids inside one workload's key space
T_W, T_X, T_A, T_B, T_DY, T_OUTLIER_MASK, T_OUTLIER_SIGN, T_MISC = range(8)

WORKLOADS = {
    "tiny": dict(seed=1, shapes=[(256, 256)], M=16, r=8, alpha=16.0, weights="normal",
                 passes="quantize+fwd+bwd"),
    "decode": dict(seed=2, shapes=[(4096, 4096)], M=(1, 4, 16), r=8, alpha=16.0,
                   weights="normal", passes="fwd"),
    "train4096": dict(seed=3, shapes=[(4096, 4096)], M=4096, r=64, alpha=16.0,
                      weights="normal", passes="quantize+fwd+bwd"),
    "llama7b": dict(seed=4, shapes=[(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)],
                    M=2048, r=64, alpha=16.0, weights="normal+outliers",
                    passes="fwd+bwd"),
    "llama65b": dict(seed=5, shapes=[(8192, 8192), (22016, 8192)], M=8192, r=64, alpha=16.0,
                     weights="student_t4", passes="fwd+bwd"),
}


def rng(seed: int, tensor_id: int, sub: int = 0) -> np.random.Generator:
    """Philox4x32-10 stream for (workload seed, tensor id, sub-index)."""
    key = np.array([seed, tensor_id * 1000003 + sub], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f32(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return (g.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def weight(seed: int, layer: int, n_out: int, k_in: int, kind: str = "normal") -> np.ndarray:
    """fp32 frozen weight W (n_out x k_in) of one layer."""
    if kind == "zero":
        return np.zeros((n_out, k_in), np.float32)
    g = rng(seed, T_W, layer)
    if kind == "normal":
        return normal_f32(g, (n_out, k_in), WEIGHT_STD)
    if kind == "normal+outliers":
        w = normal_f32(g, (n_out, k_in), WEIGHT_STD)
        gm = rng(seed, T_OUTLIER_MASK, layer)
        mask = gm.random((n_out, k_in), dtype=np.float32) < np.float32(0.001)
        gs = rng(seed, T_OUTLIER_SIGN, layer)
        sign = np.where(gs.random(int(mask.sum()), dtype=np.float32) < 0.5, -1.0, 1.0)
        w[mask] = (sign * 6.0 * WEIGHT_STD).astype(np.float32)
        return w
    if kind == "student_t4":
        # t_4 has variance nu/(nu-2) = 2; scale to std 0.02
        t = g.standard_t(4.0, size=(n_out, k_in))
        return (t * (WEIGHT_STD / np.sqrt(2.0))).astype(np.float32)
    raise ValueError(kind)


def activations(seed: int, layer: int, m: int, k: int, tensor_id: int = T_X) -> np.ndarray:
    """bf16 bits of an m x k N(0, 1) activation (X) or upstream gradient (dY)."""
    return to_bf16_bits(normal_f32(rng(seed, tensor_id, layer), (m, k), 1.0))


def lora_pair(seed: int, layer: int, n_out: int, k_in: int, r: int, b_std: float = 0.01):
    """bf16 bits of A (r x K, N(0, 1/K)) and B (N x r, N(0, b_std^2), 0.01 by default)."""
    a = to_bf16_bits(normal_f32(rng(seed, T_A, layer), (r, k_in), 1.0 / np.sqrt(k_in)))
    b = to_bf16_bits(normal_f32(rng(seed, T_B, layer), (n_out, r), b_std))
    return a, b


def layer_inputs(name: str, layer: int = 0, M: int | None = None, shape=None, r=None,
                 alpha=None, seed=None, weights: str | None = None, b_std: float = 0.01):
    """All inputs of one layer of a named workload (numpy, host).

    Returns dict(W fp32 NxK, X bf16 MxK, dY bf16 MxN, A bf16 rxK, B bf16 Nxr, alpha, r, M).
    Overrides (M, shape, r, alpha, seed) give smaller cases with the same recipe;
    ``weights`` replaces the workload's weight kind and ``b_std`` B's standard deviation.
    """
    cfg = WORKLOADS[name]
    seed = cfg["seed"] if seed is None else seed
    n_out, k_in = cfg["shapes"][layer] if shape is None else shape
    m = cfg["M"] if M is None else M
    if isinstance(m, tuple):
        m = m[-1]
    r = cfg["r"] if r is None else r
    alpha = cfg["alpha"] if alpha is None else alpha
    w = weight(seed, layer, n_out, k_in, cfg["weights"] if weights is None else weights)
    x = activations(seed, layer, m, k_in, T_X)
    dy = activations(seed, layer, m, n_out, T_DY)
    a, b = lora_pair(seed, layer, n_out, k_in, r, b_std)
    return dict(W=w, X=x, dY=dy, A=a, B=b, alpha=float(alpha), r=int(r), M=int(m),
                N=int(n_out), K=int(k_in))
