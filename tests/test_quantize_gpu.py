"""Quantizer, double quant and dequant on the GPU: bit-exact against the oracle.

Inputs follow the workloads' recipes (N(0, 0.02^2) weights, outliers, Student-t)
plus hand-built edge cases: all-zero blocks, subnormals, -0.0, exact table
values, fp32 neighbours of every decision threshold, ragged last group.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth

pytestmark = pytest.mark.gpu


def gpu_quant(W: np.ndarray):
    Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    codes, q8, s2 = q.qlora_quantize_nf4_dq(Wd)
    torch.cuda.synchronize()
    return codes, q8, s2


def check_exact(W: np.ndarray, dequant=True):
    N, K = W.shape
    codes, q8, s2 = gpu_quant(W)
    rc, rq, rs, _ = oracle.quantize_nf4_dq(W.reshape(-1))
    gc, gq, gs = codes.cpu().numpy(), q8.cpu().numpy(), s2.cpu().numpy()
    bad = np.nonzero(gc != rc)[0]
    assert bad.size == 0, f"{bad.size} code bytes differ, first at {bad[:5]}"
    assert np.array_equal(gq, rq)
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))
    if dequant:
        w32, wb = oracle.dequant(rc, rq, rs, N * K)
        d32 = q.qlora_dequant(codes, q8, s2, N, K, dtype=torch.float32).cpu().numpy().reshape(-1)
        db = q.qlora_dequant(codes, q8, s2, N, K, dtype=torch.bfloat16).view(torch.int16).cpu().numpy()
        assert np.array_equal(d32.view(np.uint32), w32.view(np.uint32))
        assert np.array_equal(db.reshape(-1).view(np.uint16), wb)
    return codes, q8, s2


def test_tiny_layer_exact():
    check_exact(synth.weight(1, 0, 256, 256))


def test_ragged_last_group_exact():
    # 3 x 6400 -> 300 blocks: one full group of 256 and a partial group of 44
    check_exact(synth.weight(11, 0, 3, 6400))
    check_exact(synth.weight(12, 0, 1, 64))          # a single block


def check_exact_single(W: np.ndarray, dequant=True):
    """Single quantization (second stage off): codes and the fp32 absmax bit-exact,
    codes identical to the double-quant call's, dense dequant bit-exact."""
    N, K = W.shape
    Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    codes, absmax = q.qlora_quantize_nf4(Wd)
    codes_dq, _, _ = q.qlora_quantize_nf4_dq(Wd)
    rc, ra = oracle.quantize_nf4(W.reshape(-1))
    gc, ga = codes.cpu().numpy(), absmax.cpu().numpy()
    assert np.array_equal(gc, rc)
    assert np.array_equal(ga.view(np.uint32), ra.view(np.uint32))
    assert torch.equal(codes, codes_dq)
    if dequant:
        w32, wb = oracle.dequant_single(rc, ra, N * K)
        d32 = q.qlora_dequant(codes, None, absmax, N, K, dtype=torch.float32).cpu().numpy().reshape(-1)
        db = q.qlora_dequant(codes, None, absmax, N, K, dtype=torch.bfloat16).view(torch.int16).cpu().numpy()
        assert np.array_equal(d32.view(np.uint32), w32.view(np.uint32))
        assert np.array_equal(db.reshape(-1).view(np.uint16), wb)


def check_exact_fp8(W: np.ndarray, dequant=True):
    """FP8 second stage: codes, q8 and s2 (sign bit included) bit-exact; codes
    identical to the linear form's; dense dequant bit-exact."""
    N, K = W.shape
    Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    codes, q8, s2 = q.qlora_quantize_nf4_dq_fp8(Wd)
    codes_lin, _, _ = q.qlora_quantize_nf4_dq(Wd)
    rc, rq, rs, _ = oracle.quantize_nf4_dq_fp8(W.reshape(-1))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(q8.cpu().numpy(), rq)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert torch.equal(codes, codes_lin)
    if dequant:
        w32, wb = oracle.dequant(rc, rq, rs, N * K)
        d32 = q.qlora_dequant(codes, q8, s2, N, K, dtype=torch.float32).cpu().numpy().reshape(-1)
        db = q.qlora_dequant(codes, q8, s2, N, K, dtype=torch.bfloat16).view(torch.int16).cpu().numpy()
        assert np.array_equal(d32.view(np.uint32), w32.view(np.uint32))
        assert np.array_equal(db.reshape(-1).view(np.uint16), wb)


def edge_case_weight():
    _, t32 = oracle.nf4_codebook()
    blocks = []
    blocks.append(np.zeros(64, np.float32))                                     # all zero
    blocks.append(np.full(64, -0.0, np.float32))                                # negative zeros
    sub = (np.arange(1, 65, dtype=np.uint32) * 977).view(np.float32)           # subnormals
    blocks.append(sub.copy())
    blocks.append(np.concatenate([sub[:32], -sub[32:]]))
    blocks.append(np.repeat(t32, 4))                                            # exact levels, absmax 1
    blocks.append(np.repeat(t32, 4) * np.float32(3.0e-3))
    blocks.append(np.repeat(t32, 4) * np.float32(-7.5))
    one = np.zeros(64, np.float32)
    one[0] = 1.0
    blocks.append(one)
    huge = np.full(64, 3.0e38, np.float32)
    huge[1::2] = -1.0e38
    blocks.append(huge)
    # fp32 neighbours of each exact midpoint, in blocks that hold -1 (absmax 1)
    probes = []
    for i in range(15):
        mid = (np.float64(t32[i]) + np.float64(t32[i + 1])) / 2
        f = np.float32(mid)
        for k in range(-20, 21):
            v = f
            for _ in range(abs(k)):
                v = np.nextafter(v, np.float32(np.inf) if k > 0 else np.float32(-np.inf))
            probes.append(v)
    probes = np.array(probes, np.float32)
    for j in range(0, probes.size, 63):
        b = np.zeros(64, np.float32)
        chunk = probes[j:j + 63]
        b[:chunk.size] = chunk
        b[63] = -1.0
        blocks.append(b)
    return np.concatenate(blocks).reshape(1, -1)


def test_edge_case_blocks_exact():
    check_exact(edge_case_weight())


def test_fp8_second_stage_exact():
    check_exact_fp8(synth.weight(1, 0, 256, 256))
    check_exact_fp8(synth.weight(11, 0, 3, 6400))              # ragged last group
    check_exact_fp8(edge_case_weight())                          # zero, subnormal, huge blocks
    check_exact_fp8(synth.weight(3, 0, 4096, 4096))
    check_exact_fp8(synth.weight(5, 0, 512, 8192, "student_t4"))  # wide spread of absmax within groups


def test_single_quant_exact():
    check_exact_single(synth.weight(1, 0, 256, 256))
    check_exact_single(synth.weight(11, 0, 3, 6400))           # ragged last group of blocks
    check_exact_single(edge_case_weight())
    check_exact_single(synth.weight(3, 0, 4096, 4096))
    check_exact_single(synth.weight(5, 0, 512, 8192, "student_t4"))


def test_all_fp32_near_every_threshold_exact():
    """Every fp32 within 2^15 ulps of each of the 15 decision midpoints (n = w exactly)."""
    _, t32 = oracle.nf4_codebook()
    vals = []
    for i in range(15):
        mid = np.float32((np.float64(t32[i]) + np.float64(t32[i + 1])) / 2)
        u = int(np.array([mid], np.float32).view(np.uint32)[0])
        mag, sign = u & 0x7FFFFFFF, u & 0x80000000
        rng = np.arange(-(1 << 15), 1 << 15, dtype=np.int64)
        v = ((mag + rng).astype(np.uint32) | np.uint32(sign)).view(np.float32)
        vals.append(v)
    vals = np.concatenate(vals).astype(np.float32)
    nb = (vals.size + 62) // 63
    W = np.zeros((nb, 64), np.float32)
    flat = np.zeros(nb * 63, np.float32)
    flat[:vals.size] = vals
    W[:, :63] = flat.reshape(nb, 63)
    W[:, 63] = -1.0
    check_exact(W.reshape(1, -1), dequant=False)


def _threshold_probe_weight(absmax_values: np.ndarray, half_width: int) -> np.ndarray:
    """Blocks whose absmax is each given value a, holding every fp32 w within half_width ulps
    of fp32(mid_i * a) for each of the 15 exact midpoints mid_i between neighbouring levels:
    fp32(w / a) then walks across every decision threshold one ulp at a time, on both sides
    of the fast path's guard band, with a reciprocal of a that is not exact."""
    _, t32 = oracle.nf4_codebook()
    mids = (t32[:-1].astype(np.float64) + t32[1:].astype(np.float64)) / 2
    offs = np.arange(-half_width, half_width, dtype=np.int64)
    rows = []
    for j, a in enumerate(absmax_values.astype(np.float32)):
        c = (mids * np.float64(a)).astype(np.float32)
        cb = c.view(np.uint32).astype(np.int64)
        probes = (cb[:, None] + offs[None, :]).astype(np.uint32).view(np.float32).reshape(-1)
        assert np.all(np.abs(probes) < a)
        nb = (probes.size + 62) // 63
        blk = np.zeros((nb, 64), np.float32)
        flat = np.zeros(nb * 63, np.float32)
        flat[:probes.size] = probes
        blk[:, :63] = flat.reshape(nb, 63)
        blk[:, 63] = a if j % 2 == 0 else -a          # the block's absmax, either sign
        rows.append(blk.reshape(-1))
    return np.concatenate(rows).reshape(1, -1)


def test_thresholds_under_inexact_reciprocals_exact():
    """~1000 block absmax values that are not powers of two, across binades from 2^-100 to
    2^100 and at both ends of a binade's mantissa range, each with every fp32 weight within
    2^12 ulps of the 15 scaled thresholds: the fast reciprocal path and its guard must give
    the codes of one IEEE division, bit for bit."""
    g = np.random.default_rng(2024)
    mant = g.uniform(1.0, 2.0, 960)
    expo = g.integers(-100, 101, 960)
    vals = [np.float32(m * 2.0 ** e) for m, e in zip(mant, expo)]
    for e in (-20, -7, -1, 0, 3):
        for m in (1.0 + 2.0 ** -23, 1.0 + 2.0 ** -22, 1.5, 2.0 - 2.0 ** -23, 2.0 - 2.0 ** -21):
            vals.append(np.float32(m * 2.0 ** e))
    vals += [np.float32(0.0173), np.float32(3 * 2.0 ** -20), np.float32(0.0731), np.float32(3.3e-3)]
    a = np.array(vals, np.float32)
    assert not np.any(np.frexp(a)[0] == 0.5)          # no power of two among them
    for part in np.array_split(a, 4):
        check_exact(_threshold_probe_weight(part, 1 << 12), dequant=False)
    check_exact(_threshold_probe_weight(a[::40], 1 << 8), dequant=True)


def test_every_fp32_in_unit_interval_exact():
    """Every fp32 n in [-1, 1] (2,130,706,434 values, zeros of both signs included), 63 to a
    block with -1.0 as the block's absmax so that w / absmax = n exactly: the GPU's codes equal
    the oracle's exact nearest-level rule on all of them.  Streamed in chunks of 2^26 weights."""
    per_chunk = (1 << 26) // 64                           # blocks per chunk
    pos = np.arange(0, 0x3F800001, dtype=np.int64)       # +0.0 .. 1.0
    total = 2 * pos.size
    done = 0
    while done < total:
        k = min(per_chunk * 63, total - done)
        idx = np.arange(done, done + k, dtype=np.int64)
        bits = np.where(idx < pos.size, idx, (idx - pos.size) | 0x80000000).astype(np.uint32)
        nb = (k + 62) // 63
        flat = np.zeros(nb * 63, np.float32)
        flat[:k] = bits.view(np.float32)
        W = np.empty((nb, 64), np.float32)
        W[:, :63] = flat.reshape(nb, 63)
        W[:, 63] = -1.0
        check_exact(W.reshape(1, -1), dequant=False)
        done += k


def test_random_fp32_in_unit_interval_exact():
    g = np.random.default_rng(123)
    bits = g.integers(0, 0x3F800001, size=(1 << 22), dtype=np.uint32)
    sign = g.integers(0, 2, size=bits.size, dtype=np.uint32) << np.uint32(31)
    vals = (bits | sign).view(np.float32)
    W = vals.reshape(-1, 64).copy()
    W[:, 0] = 1.0
    check_exact(W.reshape(64, -1), dequant=False)


def test_full_layer_4096_exact():
    check_exact(synth.weight(3, 0, 4096, 4096))


def test_outlier_and_heavy_tail_weights_exact():
    check_exact(synth.weight(4, 4, 11008, 4096, "normal+outliers")[:1024])
    check_exact(synth.weight(5, 0, 512, 8192, "student_t4"))


def test_stream_chunk_2pow26_exact():
    """One 256 MiB chunk (2^26 fp32 params) of the 65B-shaped quantize stream."""
    W = synth.weight(5, 7, 8192, 8192, "student_t4")
    check_exact(W, dequant=False)
