"""Pins for the CPU oracle: each test checks it against something other than itself.

Sources of truth used here: values the pages print (tests/golden/closed_forms.json),
two independent inverse-normal routines (Python's statistics.NormalDist and
scipy.stats.norm), exact rational arithmetic (fractions.Fraction), numpy / torch
library routines on special cases, finite differences, and algebraic identities.
"""
import json
import math
import os
from fractions import Fraction
from statistics import NormalDist

import numpy as np
import pytest
import torch
from scipy.stats import norm

import oracle
from bit_nf4_quantized_quantize_b200 import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


# --------------------------------------------------------------------- table
def test_inverse_normal_matches_two_libraries():
    ps = np.concatenate([np.logspace(-12, -1, 23), np.linspace(0.05, 0.95, 37),
                         1 - np.logspace(-12, -1, 23)])
    nd = NormalDist()
    for p in ps:
        x = oracle.norm_ppf(p)
        ref1 = nd.inv_cdf(float(p))
        ref2 = float(norm.ppf(p))
        assert abs(x - ref1) <= 1e-13 * max(1.0, abs(ref1)), (p, x, ref1)
        assert abs(x - ref2) <= 1e-13 * max(1.0, abs(ref2)), (p, x, ref2)
    assert abs(oracle.norm_ppf(0.5)) < 1e-15
    for p in (0.1, 0.3, 1 / 18, 9 / 16):
        assert abs(oracle.norm_ppf(p) + oracle.norm_ppf(1 - p)) < 1e-15


def _page_listing_table_via_scipy():
    """The codebook recipe of the page's create_nf4_codebook listing, run on scipy."""
    neg = norm.ppf(np.linspace(1 / (2 * 9), 0.5, 8, endpoint=False))
    pos = norm.ppf(np.linspace(0.5 + 1 / (2 * 8), 1 - 1 / (2 * 8), 7))
    cb = np.concatenate([neg, [0.0], pos])
    cb = cb / np.max(np.abs(cb))
    return np.sort(cb)


def _table_via_stdlib():
    nd = NormalDist()
    v = [nd.inv_cdf(i / 18) for i in range(1, 9)] + [0.0] + [nd.inv_cdf(j / 16) for j in range(9, 16)]
    mx = max(abs(a) for a in v)
    return np.sort(np.array(v) / mx)


def test_codebook_matches_independent_constructions_bitwise_in_fp32():
    t64, t32 = oracle.nf4_codebook()
    for ref in (_page_listing_table_via_scipy(), _table_via_stdlib()):
        assert np.max(np.abs(t64 - ref)) < 1e-15
        assert np.array_equal(ref.astype(np.float32).view(np.uint32), t32.view(np.uint32))
    # fp32 rounding is robust: every level sits far from an fp32 rounding boundary
    for v in t64:
        f = np.float32(v)
        if v == 0:
            continue
        ulp = np.spacing(np.abs(f))
        assert abs(float(f) - v) < 0.49 * float(ulp)


def test_codebook_invariants_from_the_pages():
    lv = GOLDEN["nf4_levels"]
    t64, t32 = oracle.nf4_codebook()
    assert t32.size == lv["total"]
    assert np.all(np.diff(t64) > 0)
    assert (t64 < 0).sum() == lv["negative"] and (t64 == 0).sum() == lv["zero"] \
        and (t64 > 0).sum() == lv["positive"]
    assert t32[0] == -1.0 and t32[8] == 0.0 and t32[15] < 1.0
    # un-normalised levels are the quantiles i/18 and j/16
    mx = abs(NormalDist().inv_cdf(1 / 18))
    for i in range(8):
        assert abs(t64[i] * mx - NormalDist().inv_cdf((i + 1) / 18)) < 1e-14
    for j in range(7):
        assert abs(t64[9 + j] * mx - NormalDist().inv_cdf((9 + j) / 16)) < 1e-14


# ------------------------------------------------------------ nearest level
def _exact_argmin(wn: float, table32):
    q = Fraction(float(wn))
    d = [abs(q - Fraction(float(c))) for c in table32]
    m = min(d)
    return d.index(m)


def test_nearest_code_is_exact_argmin_lowest_index_on_ties():
    _, t32 = oracle.nf4_codebook()
    probes = [np.float32(v) for v in np.linspace(-1, 1, 801)]
    g = np.random.default_rng(7)
    probes += [np.float32(v) for v in g.uniform(-1, 1, 400)]
    # fp32 neighbours of every exact midpoint, where a naive fp32 search can differ
    for i in range(15):
        mid = (float(t32[i]) + float(t32[i + 1])) / 2
        f = np.float32(mid)
        for k in range(-3, 4):
            v = f
            step = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
            for _ in range(abs(k)):
                v = np.nextafter(v, step)
            probes.append(np.float32(v))
    probes += [np.float32(0.0), np.float32(-0.0), np.float32(1e-40), np.float32(-1e-40),
               np.float32(1.0), np.float32(-1.0)]
    for p in probes:
        assert oracle.nearest_code(float(p), t32) == _exact_argmin(float(p), t32), p


def test_nearest_code_tie_goes_to_lower_index():
    # a table where an fp32 value lies exactly on a midpoint: levels 0.25 and 0.5
    t = np.array([-1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 0.75, 1.0] + [2.0 + i for i in range(8)],
                 np.float32)
    assert oracle.nearest_code(0.375, t) == 4
    assert oracle.nearest_code(float(np.nextafter(np.float32(0.375), np.float32(1))), t) == 5
    assert oracle.nearest_code(-0.375, t) == 1


# ----------------------------------------------------------------- quantize
def test_round_trip_of_every_table_value():
    _, t32 = oracle.nf4_codebook()
    blk = np.repeat(t32, 4).astype(np.float32)          # absmax 1 (from c_0 = -1)
    codes, absmax = oracle.quantize_nf4(blk)
    assert absmax[0] == 1.0
    unpacked = np.stack([codes & 15, codes >> 4], 1).reshape(-1)
    assert np.array_equal(unpacked, np.repeat(np.arange(16), 4))
    # with DQ: c2 = 1 -> s2 = fp32(1/255) and fp32(255 * s2) == 1 exactly
    q8, s2 = oracle.double_quant(absmax)
    assert q8[0] == 255 and s2[0] == np.float32(1) / np.float32(255)
    assert np.float32(255) * s2[0] == np.float32(1)
    w32, wb = oracle.dequant(codes, q8, s2, 64)
    assert np.array_equal(w32.view(np.uint32), blk.view(np.uint32))
    # bf16 conversion matches torch's round-to-nearest-even
    tb = torch.from_numpy(blk.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wb, tb)


def test_nibble_order_and_zero_block_and_layout():
    blk = np.zeros(128, np.float32)
    blk[0], blk[1] = -1.0, 1.0
    codes, absmax = oracle.quantize_nf4(blk)
    assert codes[0] == (0 | (15 << 4)) and codes[1] == 0x88
    assert absmax[0] == 1.0 and absmax[1] == 0.0
    assert np.all(codes[32:] == 0x88)                    # all-zero block -> level 0.0 (code 8)


def test_requantize_dequantized_codes_is_identity():
    _, t32 = oracle.nf4_codebook()
    g = np.random.default_rng(3)
    nblk = 512
    codes = g.integers(0, 16, size=(nblk, 64))
    codes[:, g.integers(0, 64, nblk)] = 0                # every block holds code 0 -> absmax
    codes[np.arange(nblk), g.integers(0, 64, nblk)] = 0
    scale = g.uniform(1e-3, 10.0, nblk).astype(np.float32)
    w = (t32[codes] * scale[:, None]).astype(np.float32).reshape(-1)
    c2, am = oracle.quantize_nf4(w)
    un = np.stack([c2 & 15, c2 >> 4], 1).reshape(nblk, 64)
    assert np.array_equal(un, codes)
    assert np.array_equal(am, scale)


def test_power_of_two_scaling_is_exact():
    x = synth.normal_f32(synth.rng(9, 0), (64 * 40,), 0.02)
    c1, a1 = oracle.quantize_nf4(x)
    for e in (-20, -3, 5, 30):
        c2, a2 = oracle.quantize_nf4((x * np.float32(2.0 ** e)).astype(np.float32))
        assert np.array_equal(c1, c2)
        assert np.array_equal(a2, (a1 * np.float32(2.0 ** e)).astype(np.float32))


def test_quantize_brute_force_tiny():
    """Brute force over all 16 levels with exact rationals on the tiny workload's first rows."""
    _, t32 = oracle.nf4_codebook()
    w = synth.weight(1, 0, 256, 256)[:4].reshape(-1)     # 1024 values, 16 blocks
    codes, absmax = oracle.quantize_nf4(w)
    un = np.stack([codes & 15, codes >> 4], 1).reshape(-1)
    for b in range(w.size // 64):
        blk = w[b * 64:(b + 1) * 64]
        am = max(abs(float(v)) for v in blk)
        assert absmax[b] == np.float32(am)
        for j, v in enumerate(blk):
            n = np.float32(v) / np.float32(am)           # IEEE fp32 division (numpy)
            assert un[b * 64 + j] == _exact_argmin(float(n), t32)


def test_nf4_beats_int4_on_normal_data():
    """Sanity from the pages: NF4's MSE is roughly 10-30% below uniform INT4 (N(0,1), block 64)."""
    spec = GOLDEN["nf4_vs_int4_mse_improvement_percent"]
    g = synth.rng(42, 0)
    w = g.standard_normal(spec["samples"] - spec["samples"] % 64).astype(np.float32)
    codes, absmax = oracle.quantize_nf4(w)
    _, t32 = oracle.nf4_codebook()
    un = np.stack([codes & 15, codes >> 4], 1).reshape(-1)
    w_nf4 = t32[un].astype(np.float64) * np.repeat(absmax.astype(np.float64), 64)
    lv = np.linspace(-1, 1, 16)
    wb = w.reshape(-1, 64).astype(np.float64)
    am = np.abs(wb).max(1, keepdims=True)
    idx = np.abs(wb[:, :, None] / am[:, :, None] - lv[None, None, :]).argmin(-1)
    w_int4 = (lv[idx] * am).reshape(-1)
    mse_nf4 = np.mean((w - w_nf4) ** 2)
    mse_int4 = np.mean((w - w_int4) ** 2)
    imp = 100 * (1 - mse_nf4 / mse_int4)
    assert spec["low"] - 5 <= imp <= spec["high"] + 5, imp


# ---------------------------------------------------------- double quant
def test_double_quant_hand_cases():
    c2 = np.float32(0.037)
    a = np.array([c2] * 256, np.float32)
    q8, s2 = oracle.double_quant(a)
    assert np.all(q8 == 255) and s2[0] == c2 / np.float32(255)
    a = np.zeros(256, np.float32)
    a[0], a[1] = c2, c2 / np.float32(2)
    q8, s2 = oracle.double_quant(a)
    s = Fraction(float(s2[0]))
    half = Fraction(float(np.float32(np.float32(c2 / np.float32(2)) / s2[0])))
    exp = int(half.__round__())                           # Fraction rounds half to even
    assert q8[0] == 255 and q8[1] == exp and np.all(q8[2:] == 0)
    assert s == Fraction(float(np.float32(c2) / np.float32(255)))


def test_double_quant_error_bound_and_partial_group():
    g = np.random.default_rng(11)
    a = np.abs(g.normal(0, 0.05, 256 * 7 + 100)).astype(np.float32)   # ragged last group
    q8, s2 = oracle.double_quant(a)
    assert s2.size == 8
    for i, v in enumerate(a):
        s = float(s2[i // 256])
        rec = float(np.float32(np.float32(q8[i]) * s2[i // 256]))
        assert abs(rec - float(v)) <= s / 2 * (1 + 1e-6) + 1e-12
        grp = a[(i // 256) * 256:(i // 256 + 1) * 256]
        assert s2[i // 256] == np.float32(grp.max()) / np.float32(255)


def test_double_quant_zero_and_subnormal_groups():
    q8, s2 = oracle.double_quant(np.zeros(256, np.float32))
    assert s2[0] == 0 and np.all(q8 == 0)
    tiny = np.full(256, np.float32(1e-44), np.float32)    # c2/255 underflows to 0
    q8, s2 = oracle.double_quant(tiny)
    assert s2[0] == 0 and np.all(q8 == 0)


# --------------------------------------------------- FP8 reading of the DQ
def _torch_e4m3_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_every_code_matches_torch():
    codes = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(oracle.e4m3_to_f32(codes).view(np.uint32), ref.view(np.uint32))


def test_e4m3_encode_is_round_to_nearest_even_and_saturates():
    g = np.random.default_rng(31)
    x = np.concatenate([g.uniform(0, 448, 3000), 2.0 ** g.uniform(-12, 8.8, 3000)]).astype(np.float32)
    # exact midpoints between neighbouring E4M3 values (ties go to the even mantissa)
    vals = oracle.e4m3_to_f32(np.arange(0, 0x7E, dtype=np.uint8)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, vals.astype(np.float32)])
    x = x[x <= 448]
    assert np.array_equal(oracle.f32_to_e4m3(x), _torch_e4m3_bits(x))
    # above the largest finite value the conversion saturates to 448 (code 0x7E)
    assert np.all(oracle.f32_to_e4m3(np.array([448.5, 463.9, 464.0, 470.0, 1e30], np.float32)) == 0x7E)


def test_double_quant_fp8_cases_and_error_bound():
    # a group of equal constants: every q is 448's code and fp32(448 * |s2|) is within 1 ulp of c2
    a = np.full(256, 0.37, np.float32)
    q8, s2 = oracle.double_quant_fp8(a)
    assert np.all(q8 == 0x7E) and np.signbit(s2[0])
    assert abs(np.float32(448) * -s2[0] - np.float32(0.37)) <= np.spacing(np.float32(0.37))
    # zero group: q = 0, s2 = -0.0, dequant 0
    q8, s2 = oracle.double_quant_fp8(np.zeros(300, np.float32))
    assert np.all(q8 == 0) and np.all(s2 == 0) and np.all(np.signbit(s2))
    # random constants: relative error <= 2^-4 in E4M3's normal range, <= 2^-10 |s2| below it
    g = np.random.default_rng(32)
    a = (2.0 ** g.uniform(-20, 0, 256 * 40)).astype(np.float32)
    q8, s2 = oracle.double_quant_fp8(a)
    s = np.repeat(-s2, 256)[: a.size].astype(np.float64)
    c1 = (oracle.e4m3_to_f32(q8).astype(np.float32) * s.astype(np.float32)).astype(np.float64)
    ratio = a / s
    err = np.abs(c1 - a)
    normal = ratio >= 2.0 ** -6
    assert np.all(err[normal] <= a[normal] * 2.0 ** -4 * (1 + 1e-6))
    assert np.all(err[~normal] <= s[~normal] * 2.0 ** -10 * (1 + 1e-6))


def test_dequant_fp8_matches_formula_in_numpy():
    w = synth.weight(2, 0, 512, 512).reshape(-1)
    codes, absmax = oracle.quantize_nf4(w)
    q8, s2 = oracle.double_quant_fp8(absmax)
    _, t32 = oracle.nf4_codebook()
    w32, wb = oracle.dequant(codes, q8, s2, w.size)
    un = np.stack([codes & 15, codes >> 4], 1).reshape(-1)
    qv = torch.from_numpy(q8.copy()).view(torch.float8_e4m3fn).float().numpy()
    c1 = (qv * np.repeat(-s2, 256)[: q8.size]).astype(np.float32)
    ref = (t32[un] * np.repeat(c1, 64)).astype(np.float32)
    assert np.array_equal(w32.view(np.uint32), ref.view(np.uint32))
    # the 8-bit codes cost the same 4.127 bit/param as the linear format
    assert 8 * (codes.nbytes + q8.nbytes + s2.nbytes) / w.size == 4 + 8 / 64 + 32 / (64 * 256)


# ---------------------------------------------------------------- overhead
def test_overheads_match_the_pages_closed_forms():
    G = GOLDEN
    sq = 32 / 64
    dq = 4 + 8 / 64 + 32 / (64 * 256)
    assert sq == G["single_quant_overhead_bit_per_param"]["value"]
    assert 4 + sq == G["single_quant_total_bit_per_param"]["value"]
    assert 8 / 64 == G["double_quant_second_term_bit_per_param"]["value"]
    assert abs(32 / (64 * 256) - G["double_quant_third_term_bit_per_param_approx"]["value"]) \
        <= G["double_quant_third_term_bit_per_param_approx"]["tolerance_abs"]
    assert abs(dq - G["double_quant_total_bit_per_param_approx"]["value"]) <= 5e-4
    saving = 4.5 - dq
    assert saving == 0.373046875
    assert abs(saving - G["dq_saving_bit_per_param_approx"]["value"]) <= 5e-3
    assert abs(65e9 * sq / 8 / 1e9 - 4.0) <= 0.1
    assert abs(65e9 * saving / 8 / 1e9 - 3.0) <= 0.1
    # the buffers the oracle produces have exactly that size, for every workload shape
    for shape in [(256, 256), (4096, 4096), (11008, 4096), (4096, 11008), (8192, 8192),
                  (22016, 8192)]:
        n = shape[0] * shape[1]
        nb = n // 64
        bytes_ = n // 2 + nb + 4 * ((nb + 255) // 256)
        assert 8 * bytes_ / n == dq
    w = synth.weight(1, 0, 256, 256)
    codes, q8, s2, _ = oracle.quantize_nf4_dq(w.reshape(-1))
    assert 8 * (codes.nbytes + q8.nbytes + s2.nbytes) / w.size == dq


def test_lora_parameter_counts():
    G = GOLDEN
    d = k = 4096
    assert 8 * (d + k) == G["lora_params_d4096_k4096_r8"]["value"]
    assert d * k == G["dense_params_d4096_k4096"]["value"]
    assert abs(100 * 8 * (d + k) / (d * k) - 0.4) <= 0.05
    assert 4 * 2 * 4096 * 64 * 32 == G["lora_params_7b_attention_r64"]["value"]


# --------------------------------------------------------------- bf16 / dequant
def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(5)
    x = np.concatenate([g.normal(0, 1, 5000), g.normal(0, 1e-30, 200), [0.0, -0.0, 1e38, -3e-39]])
    x = x.astype(np.float32)
    # values exactly halfway between two bf16 numbers (tie -> even)
    ties = (np.arange(1, 200, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32) + 0])
    ours = oracle.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_dequant_matches_formula_in_fp32_numpy():
    w = synth.weight(1, 0, 256, 256).reshape(-1)
    codes, q8, s2, _ = oracle.quantize_nf4_dq(w)
    _, t32 = oracle.nf4_codebook()
    w32, wb = oracle.dequant(codes, q8, s2, w.size)
    un = np.stack([codes & 15, codes >> 4], 1).reshape(-1)
    c1 = (q8.astype(np.float32) * np.repeat(s2, 256)[: q8.size]).astype(np.float32)
    ref = (t32[un] * np.repeat(c1, 64)).astype(np.float32)
    assert np.array_equal(w32.view(np.uint32), ref.view(np.uint32))
    tb = torch.from_numpy(ref.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wb, tb)
    # reconstruction error: within half a level spacing times absmax plus the DQ error
    assert np.max(np.abs(w32 - w)) < 0.2 * np.abs(w).max()


# ------------------------------------------------------- single quantization
def test_single_quant_round_trip_and_size():
    """First stage only (p1 §5-2 memory arithmetic, Single Q): the block scale is
    absmax itself, so table values times a power of two come back bit-exactly,
    and the stored buffers come to the printed 4 + 32/64 = 4.5 bit/param."""
    _, t32 = oracle.nf4_codebook()
    blk = np.repeat(t32, 4).astype(np.float32)
    for e in (-7, 0, 9):
        x = (blk * np.float32(2.0 ** e)).astype(np.float32)
        codes, absmax = oracle.quantize_nf4(x)
        assert absmax[0] == np.float32(2.0 ** e)
        w32, wb = oracle.dequant_single(codes, absmax, 64)
        assert np.array_equal(w32.view(np.uint32), x.view(np.uint32))
        tb = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(wb, tb)
    w = synth.weight(1, 0, 256, 256).reshape(-1)
    codes, absmax = oracle.quantize_nf4(w)
    assert 8 * (codes.nbytes + absmax.nbytes) / w.size == GOLDEN["single_quant_total_bit_per_param"]["value"]


def test_single_quant_dequant_formula_and_error_bound():
    """Independent fp32 restatement in numpy, bf16 against torch, and the
    reconstruction error within half the widest level gap times absmax."""
    w = synth.weight(3, 0, 512, 512).reshape(-1)
    codes, absmax = oracle.quantize_nf4(w)
    _, t32 = oracle.nf4_codebook()
    w32, wb = oracle.dequant_single(codes, absmax, w.size)
    un = np.stack([codes & 15, codes >> 4], 1).reshape(-1)
    ref = (t32[un] * np.repeat(absmax, 64)).astype(np.float32)
    assert np.array_equal(w32.view(np.uint32), ref.view(np.uint32))
    tb = torch.from_numpy(ref.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wb, tb)
    half_gap = np.max(np.diff(t32.astype(np.float64))) / 2
    err = np.abs(w32.astype(np.float64) - w) / np.repeat(absmax, 64).astype(np.float64)
    assert np.max(err) <= half_gap * (1 + 1e-6)


def test_single_and_double_quant_agree_when_dq_is_exact():
    """When every absmax of a group equals the group maximum and that maximum is
    a power of two, fp32(255 * fp32(c2/255)) == c2, so the two-level scale is
    the absmax itself and both dequantizations give the same bits."""
    g = np.random.default_rng(11)
    nblk = 256
    codes = g.integers(0, 16, size=(nblk, 64))
    codes[:, 0] = 0                                     # every block holds level -1 -> absmax = scale
    _, t32 = oracle.nf4_codebook()
    for e in (-12, 0, 3):
        sc = np.float32(2.0 ** e)
        w = (t32[codes] * sc).astype(np.float32).reshape(-1)
        c, q8, s2, absmax = oracle.quantize_nf4_dq(w)
        assert np.all(absmax == sc) and np.all(q8 == 255)
        a, ab = oracle.dequant(c, q8, s2, w.size)
        b, bb = oracle.dequant_single(c, absmax, w.size)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)) and np.array_equal(ab, bb)


# ---------------------------------------------------------- adapter merge
def _bf16_exact_nearest(x: float) -> int:
    """bf16 bits nearest to x (ties to even), by exact rational comparison of the
    two bf16 neighbours of x (finite bf16 range)."""
    from fractions import Fraction
    fx = Fraction(x)
    if fx == 0:
        return 0x8000 if np.signbit(x) else 0
    sign = 0x8000 if fx < 0 else 0
    a = abs(fx)
    # candidates: every bf16 magnitude whose fp32 value brackets a
    lo_bits = int(np.array([np.float32(float(a))], np.float32).view(np.uint32)[0]) >> 16
    cands = [b for b in (lo_bits - 1, lo_bits, lo_bits + 1, lo_bits + 2) if 0 <= b < 0x7F80]
    val = lambda b: Fraction(float(np.array([b << 16], np.uint32).view(np.float32)[0]))
    best = min(cands, key=lambda b: (abs(val(b) - a), b & 1))
    return sign | best


def test_f64_to_bf16_is_nearest_ties_to_even():
    g = np.random.default_rng(21)
    xs = list(g.normal(0, 1, 3000)) + list(g.normal(0, 1e-30, 300)) + list(g.normal(0, 1e30, 300))
    # exact ties between two bf16 values, and points one fp64 ulp either side
    for b in g.integers(0x0080, 0x7F00, 300):
        lo = float(np.array([int(b) << 16], np.uint32).view(np.float32)[0])
        hi = float(np.array([(int(b) + 1) << 16], np.uint32).view(np.float32)[0])
        mid = (lo + hi) / 2
        xs += [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf), -mid]
    xs = np.array(xs, np.float64)
    ours = oracle.f64_to_bf16_bits(xs)
    ref = np.array([_bf16_exact_nearest(float(x)) for x in xs], np.uint16)
    assert np.array_equal(ours, ref)
    # fp32-exact inputs agree with torch's fp32 -> bf16 rounding
    x32 = g.normal(0, 1, 2000).astype(np.float32)
    tb = torch.from_numpy(x32.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16_bits(x32.astype(np.float64)), tb)


def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


def test_merge_adapter_zero_b_is_the_bf16_base():
    """[p4] merge into the 16-bit base: with B = 0 the merged weight is bf16(W)."""
    W = synth.weight(1, 0, 64, 128)
    A = _bf16_bits(np.random.default_rng(1).normal(0, 0.1, (8, 128)))
    B = np.zeros((64, 8), np.uint16)
    assert np.array_equal(oracle.merge_adapter(W, A, B, 16.0), _bf16_bits(W))


def test_merge_adapter_exact_rational_cases():
    """Dyadic inputs of moderate range keep every fp64 step exact, so the merged
    weight is the exact value bf16(W) + s B A rounded once (Fraction arithmetic)."""
    from fractions import Fraction
    g = np.random.default_rng(5)
    N, K, r, alpha = 12, 40, 4, 16.0              # s = 4, a power of two
    W = (g.integers(-64, 65, (N, K)) / 64.0).astype(np.float32)
    A = _bf16_bits(g.integers(-32, 33, (r, K)) / 128.0)
    B = _bf16_bits(g.integers(-32, 33, (N, r)) / 1024.0)
    out = oracle.merge_adapter(W, A, B, alpha)
    Af, Bf = _bits_to_f64(A), _bits_to_f64(B)
    s = Fraction(alpha) / r
    for n in range(N):
        for k in range(K):
            v = Fraction(float(W[n, k])) + s * sum(Fraction(Bf[n, j]) * Fraction(Af[j, k]) for j in range(r))
            assert out[n, k] == _bf16_exact_nearest(float(v)), (n, k)


def test_merge_adapter_layer_identity():
    """X merged^T equals X bf16(W)^T + s (X A^T) B^T up to the one bf16 rounding of the merge."""
    g = np.random.default_rng(8)
    N, K, M, r, alpha = 96, 192, 5, 8, 16.0
    W = synth.weight(2, 0, N, K)
    Ab = _bf16_bits(g.normal(0, 1 / np.sqrt(K), (r, K)))
    Bb = _bf16_bits(g.normal(0, 0.5, (N, r)))
    Wm = _bits_to_f64(oracle.merge_adapter(W, Ab, Bb, alpha))
    X = g.normal(size=(M, K))
    s = np.float64(np.float32(alpha / r))
    ref = X @ _bits_to_f64(_bf16_bits(W)).T + s * (X @ _bits_to_f64(Ab).T) @ _bits_to_f64(Bb).T
    got = X @ Wm.T
    # each merged element is within half a bf16 ulp (2^-9 relative) of its exact value
    bound = np.abs(X) @ (np.abs(Wm).T * 2.0 ** -8)
    assert np.all(np.abs(got - ref) <= bound + 1e-12)


# ------------------------------------------------------------- LoRA dropout
def test_philox_known_answers():
    kat = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        h = lambda xs: np.array([int(x, 16) for x in xs], np.uint32)
        assert np.array_equal(oracle.philox4x32_10(h(v["counter"]), h(v["key"])), h(v["out"]))


def test_dropout_keep_rate_and_layout():
    M, K = 512, 2048
    for p in (0.05, 0.5):
        keep = oracle.dropout_keep(M, K, p, seed=1234, offset=7)
        n = keep.size
        assert abs(keep.mean() - (1 - p)) <= 5 * np.sqrt(p * (1 - p) / n)
    assert np.all(oracle.dropout_keep(8, 64, 0.0, seed=1, offset=0) == 1)
    # 16-bit thresholds: floor(p * 2^16) of the fp32 p; the largest fp32 below 1 gives 2^16 - 1
    assert oracle.dropout_threshold(0.25) == 16384 and oracle.dropout_threshold(0.05) == 3276
    assert oracle.dropout_threshold(float(np.nextafter(np.float32(1), np.float32(0)))) == 65535
    # element e = m*K + k uses the 16-bit half e & 1 (low half first) of word (e >> 1) & 3 of
    # the block at counter (e >> 3, offset)
    keep = oracle.dropout_keep(4, 64, 0.25, seed=0x1122334455667788, offset=0x99)
    t = oracle.dropout_threshold(0.25)
    for e in (0, 1, 2, 3, 4, 5, 6, 7, 8, 77, 255):
        w = oracle.philox4x32_10([e >> 3, 0, 0x99, 0], [0x55667788, 0x11223344])
        half = (int(w[(e >> 1) & 3]) >> (16 * (e & 1))) & 0xFFFF
        assert keep.reshape(-1)[e] == (1 if half >= t else 0)
    # another offset gives another mask
    assert not np.array_equal(oracle.dropout_keep(64, 64, 0.5, 3, 0), oracle.dropout_keep(64, 64, 0.5, 3, 1))


def test_dropout_with_p_zero_is_the_plain_layer():
    X, W, A, B, dY = _small_case()
    keep = np.ones_like(X, dtype=np.uint8)
    Y0, U0 = oracle.linear_fwd(X, W, A, B, 5.0)
    Y1, U1 = oracle.linear_fwd_dropout(X, W, A, B, 5.0, keep, 0.0)
    assert np.allclose(Y0, Y1, rtol=1e-13, atol=1e-13) and np.allclose(U0, U1, rtol=1e-13, atol=1e-13)
    for a, b in zip(oracle.linear_bwd(X, W, A, B, dY, 5.0), oracle.linear_bwd_dropout(X, W, A, B, dY, 5.0, keep, 0.0)):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_dropout_bwd_against_finite_differences():
    """With the mask fixed, L = <dY, Y> is smooth in A, B and X: central differences
    check every gradient formula, including the masked adapter term of dX."""
    X, W, A, B, dY = _small_case(M=6, N=10, K=64, r=3, seed=4)
    p = 0.3
    keep = oracle.dropout_keep(6, 64, p, seed=9, offset=0)
    alpha = 4.0
    L = lambda X_, A_, B_: float(np.sum(dY * oracle.linear_fwd_dropout(X_, W, A_, B_, alpha, keep, p)[0]))
    dX, dA, dB = oracle.linear_bwd_dropout(X, W, A, B, dY, alpha, keep, p)
    h = 1e-6
    for name, arr, grad in (("A", A, dA), ("B", B, dB), ("X", X, dX)):
        g = np.random.default_rng(0)
        for _ in range(12):
            idx = tuple(g.integers(0, d) for d in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args = {"A": (X, plus, B), "B": (X, A, plus), "X": (plus, A, B)}[name]
            argm = {"A": (X, minus, B), "B": (X, A, minus), "X": (minus, A, B)}[name]
            num = (L(*args) - L(*argm)) / (2 * h)
            assert abs(num - grad[idx]) <= 1e-6 * max(1.0, abs(num)), (name, idx, num, grad[idx])


def test_dropout_hand_case_at_p_half():
    """Two tokens, K = N = 2, r = 1, alpha = 1 (s = 1), p = 0.5 (1/(1-p) = 2) and a fixed mask,
    worked by hand from the PEFT LoRA layer (dropout on the adapter input only):
    Xd = 2 X*keep = [[2, 0], [0, -2]], U = Xd A^T = [2, -2], X W^T = [[-1, 4], [5, 1]],
    s U B^T = [[8, -2], [-8, 2]]; V = dY B = [4, -1], dY W = [[2, -1], [1, 1]],
    2 (V A)*keep = [[8, 0], [0, -2]], dA = s V^T Xd = [8, 2], dB = s dY^T U = [2, -2].
    A missing or inverted 1/(1-p), a mask on the frozen path, or an unmasked dX adapter term
    each change these numbers."""
    X = np.array([[1.0, 3.0], [2.0, -1.0]])
    keep = np.array([[1, 0], [0, 1]], np.uint8)
    W = np.array([[2.0, -1.0], [1.0, 1.0]])
    A = np.array([[1.0, 1.0]])
    B = np.array([[4.0], [-1.0]])
    dY = np.array([[1.0, 0.0], [0.0, 1.0]])
    Y, U = oracle.linear_fwd_dropout(X, W, A, B, 1.0, keep, 0.5)
    assert np.array_equal(U, [[2.0], [-2.0]])
    assert np.array_equal(Y, [[7.0, 2.0], [-3.0, 3.0]])
    dX, dA, dB = oracle.linear_bwd_dropout(X, W, A, B, dY, 1.0, keep, 0.5)
    assert np.array_equal(dX, [[10.0, -1.0], [1.0, -1.0]])
    assert np.array_equal(dA, [[8.0, 2.0]])
    assert np.array_equal(dB, [[2.0], [-2.0]])


def test_dropout_exact_rational_case_at_p_half():
    """Dyadic inputs and a Philox mask at p = 0.5: every product and sum is exact in fp64, so
    the oracle must equal exact rational arithmetic of Y = X W^T + s (2 X*keep) A^T B^T and of
    its gradients, written element by element."""
    g = np.random.default_rng(11)
    M, N, K, r, alpha = 3, 4, 64, 2, 6.0
    X = g.integers(-8, 9, (M, K)) / 4.0
    W = g.integers(-8, 9, (N, K)) / 8.0
    A = g.integers(-4, 5, (r, K)) / 16.0
    B = g.integers(-4, 5, (N, r)) / 2.0
    dY = g.integers(-4, 5, (M, N)) / 2.0
    keep = oracle.dropout_keep(M, K, 0.5, seed=5, offset=1)
    assert 0 < keep.sum() < keep.size
    F = Fraction
    s = F(alpha) / r
    Xd = [[F(X[m, k]) * keep[m, k] * 2 for k in range(K)] for m in range(M)]
    U = [[sum(Xd[m][k] * F(A[j, k]) for k in range(K)) for j in range(r)] for m in range(M)]
    V = [[sum(F(dY[m, n]) * F(B[n, j]) for n in range(N)) for j in range(r)] for m in range(M)]
    Yq = [[sum(F(X[m, k]) * F(W[n, k]) for k in range(K)) + s * sum(U[m][j] * F(B[n, j]) for j in range(r))
           for n in range(N)] for m in range(M)]
    dXq = [[sum(F(dY[m, n]) * F(W[n, k]) for n in range(N))
            + s * sum(V[m][j] * F(A[j, k]) for j in range(r)) * keep[m, k] * 2 for k in range(K)] for m in range(M)]
    dAq = [[s * sum(V[m][j] * Xd[m][k] for m in range(M)) for k in range(K)] for j in range(r)]
    dBq = [[s * sum(F(dY[m, n]) * U[m][j] for m in range(M)) for j in range(r)] for n in range(N)]
    Y, Uo = oracle.linear_fwd_dropout(X, W, A, B, alpha, keep, 0.5)
    dX, dA, dB = oracle.linear_bwd_dropout(X, W, A, B, dY, alpha, keep, 0.5)
    for got, want in ((Y, Yq), (Uo, U), (dX, dXq), (dA, dAq), (dB, dBq)):
        assert [[F(v) for v in row] for row in got.tolist()] == want


def test_dropout_leaves_the_frozen_path_unmasked():
    """B = 0 removes the adapter from Y, and A = 0 removes it from dX: whatever the mask, the
    frozen product X W^T (and dY W) must come out unmasked and unscaled (numpy matmul)."""
    X, W, A, B, dY = _small_case(M=6, N=10, K=64, r=3, seed=8)
    for p in (0.3, 0.5, 0.9):
        keep = oracle.dropout_keep(6, 64, p, seed=3, offset=2)
        assert keep.sum() < keep.size
        Y, U = oracle.linear_fwd_dropout(X, W, A, np.zeros_like(B), 4.0, keep, p)
        assert np.allclose(Y, X @ W.T, rtol=1e-13, atol=1e-13)
        dX, _, _ = oracle.linear_bwd_dropout(X, W, np.zeros_like(A), B, dY, 4.0, keep, p)
        assert np.allclose(dX, dY @ W, rtol=1e-13, atol=1e-13)


def _nearest_f32(q: Fraction) -> float:
    """Exact rational -> nearest fp32 (ties to even), for positive normal values."""
    e = math.floor(math.log2(q))
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    scaled = q / Fraction(2) ** (e - 23)          # in [2^23, 2^24)
    m = math.floor(scaled)
    rem = scaled - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    return float(np.float32(m * 2.0 ** (e - 23)))


def test_dropout_scale_on_its_own():
    """The kept-input scale is 1/(1 - p) of the fp32 p, rounded once to fp32 (exact rational
    check), and it makes the masked input unbiased: the mean of X*keep*scale over 2^20 ones is
    1 within the binomial bound (a (1 - p) factor, or none, would miss by p or more)."""
    for p in (0.05, 0.1, 0.3, 0.5, 0.75, 0.999):
        p32 = Fraction(float(np.float32(p)))
        assert oracle.dropout_scale(p) == _nearest_f32(1 / (1 - p32)), p
    assert oracle.dropout_scale(0.5) == 2.0 and oracle.dropout_scale(0.75) == 4.0
    for p in (0.05, 0.5):
        keep = oracle.dropout_keep(1024, 1024, p, seed=21, offset=0)
        n = keep.size
        mean = float(keep.mean()) * oracle.dropout_scale(p)
        keep_rate = 1 - oracle.dropout_threshold(p) / 65536.0
        assert abs(mean - keep_rate * oracle.dropout_scale(p)) <= 5 * np.sqrt(p * (1 - p) / n) * oracle.dropout_scale(p)
        assert abs(mean - 1.0) <= 5 * np.sqrt(p * (1 - p) / n) * oracle.dropout_scale(p) + 2.0 ** -15
        X = np.ones((4, 64))
        Y, U = oracle.linear_fwd_dropout(X, np.zeros((1, 64)), np.ones((1, 64)), np.zeros((1, 1)), 1.0,
                                         keep[:4, :64], p)
        assert np.allclose(U[:, 0], keep[:4, :64].sum(axis=1) * oracle.dropout_scale(p), rtol=1e-15)


# ----------------------------------------------------------------- linear
def _small_case(M=9, N=24, K=64, r=3, seed=0):
    g = np.random.default_rng(seed)
    return (g.normal(size=(M, K)), g.normal(size=(N, K)) * 0.1, g.normal(size=(r, K)) / 8,
            g.normal(size=(N, r)) * 0.1, g.normal(size=(M, N)))


def test_fwd_special_cases_and_merge_identity():
    X, W, A, B, _ = _small_case()
    alpha = 5.0
    s = alpha / A.shape[0]
    Y, U = oracle.linear_fwd(X, W, A, np.zeros_like(B), alpha)
    assert np.allclose(Y, X @ W.T, rtol=1e-13, atol=1e-13)
    Y, U = oracle.linear_fwd(X, W, A, B, alpha)
    # merging the adapter into the dense weight gives the same layer
    assert np.allclose(Y, X @ (W + s * B @ A).T, rtol=1e-12, atol=1e-12)
    assert np.allclose(U, X @ A.T, rtol=1e-13, atol=1e-13)
    rows = np.array([7, 0, 3])
    Yr, Ur = oracle.linear_fwd(X, W, A, B, alpha, rows=rows)
    assert np.array_equal(Yr, Y[rows]) and np.array_equal(Ur, U[rows])


def test_bwd_against_finite_differences_and_adjoint():
    X, W, A, B, dY = _small_case(M=5, N=8, K=6, r=2, seed=1)
    alpha = 3.0

    def loss(A_, B_, X_=X):
        return float(np.sum(dY * oracle.linear_fwd(X_, W, A_, B_, alpha)[0]))

    dX, dA, dB = oracle.linear_bwd(X, W, A, B, dY, alpha)
    h = 1e-6
    for idx in np.ndindex(A.shape):
        Ap, Am = A.copy(), A.copy()
        Ap[idx] += h
        Am[idx] -= h
        assert abs((loss(Ap, B) - loss(Am, B)) / (2 * h) - dA[idx]) < 1e-7
    for idx in np.ndindex(B.shape):
        Bp, Bm = B.copy(), B.copy()
        Bp[idx] += h
        Bm[idx] -= h
        assert abs((loss(A, Bp) - loss(A, Bm)) / (2 * h) - dB[idx]) < 1e-7
    for idx in [(0, 0), (2, 3), (4, 5)]:
        Xp, Xm = X.copy(), X.copy()
        Xp[idx] += h
        Xm[idx] -= h
        assert abs((loss(A, B, Xp) - loss(A, B, Xm)) / (2 * h) - dX[idx]) < 1e-7
    # the layer is linear in X: <dY, Y(X)> == <dX, X>
    Y, _ = oracle.linear_fwd(X, W, A, B, alpha)
    assert abs(np.sum(dY * Y) - np.sum(dX * X)) < 1e-10 * max(1, abs(np.sum(dY * Y)))


def test_bwd_zero_adapter_and_rows():
    X, W, A, B, dY = _small_case(M=7, N=16, K=64, r=4, seed=2)
    dX, dA, dB = oracle.linear_bwd(X, W, A, np.zeros_like(B), dY, 8.0)
    assert np.allclose(dX, dY @ W, rtol=1e-13, atol=1e-13)
    assert np.all(dA == 0)
    assert np.allclose(dB, 2.0 * dY.T @ (X @ A.T), rtol=1e-12, atol=1e-12)
    dX, dA, dB = oracle.linear_bwd(X, W, A, B, dY, 8.0)
    dXr, dAr, dBr = oracle.linear_bwd(X, W, A, B, dY, 8.0, rows=np.array([6, 1]))
    assert np.array_equal(dXr, dX[[6, 1]]) and np.array_equal(dAr, dA) and np.array_equal(dBr, dB)


def test_oracle_rejects_ragged_length():
    with pytest.raises(ValueError):
        oracle.quantize_nf4(np.zeros(65, np.float32))


def test_planted_mistake_is_caught():
    """A plausible slip (dropping the alpha/r scale on the adapter) fails the merge identity."""
    X, W, A, B, _ = _small_case()
    Y, _ = oracle.linear_fwd(X, W, A, B, 5.0)
    wrong = X @ (W + B @ A).T
    assert not np.allclose(Y, wrong, rtol=1e-6, atol=1e-6)
