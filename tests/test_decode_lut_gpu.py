"""Few-token forward on the table-lookup path (one to four tokens) against the fp64 oracle.

The cases exercise that kernel's own logic: the activations' block-wise power-of-two
scaling to fp16 at extreme and mixed magnitudes, K ranges that do not split evenly over
the 16 warps (tail blocks, idle warps), tiles streamed through a ring with fewer slots
than tiles (one and two slots), single quantization and the FP8 second stage, wide
adapters, and run-to-run determinism.  The forward is checked with the same bounds as
every other path (rel-L2 <= 4e-3 and the element-wise bound of tests/common.py).
"""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth
from common import to_dev_bf16
from test_linear_gpu import run_case

pytestmark = pytest.mark.gpu


def _scaled_x(inp, fn):
    """Replace X by fn(X as fp32, row index) rounded to bf16."""
    x = synth.bf16_bits_to_f32(inp["X"]).astype(np.float64)
    for t in range(x.shape[0]):
        x[t] = fn(x[t], t)
    inp["X"] = synth.to_bf16_bits(x.astype(np.float32))
    return inp


@pytest.mark.parametrize("kind", ["large", "small", "outlier", "zero_token", "log_uniform"])
def test_activation_magnitudes(kind):
    """Each 64-column block of a token is scaled by its own power of two before the fp16
    conversion; results must not depend on the activations' overall magnitude."""
    inp = synth.layer_inputs("tiny", M=4, shape=(512, 2048), r=8, seed=1300)
    rng = np.random.default_rng(1301)
    if kind == "large":
        fn = lambda v, t: v * 2.0 ** (40 + 10 * t)       # up to 2^70, far above fp16's range
    elif kind == "small":
        fn = lambda v, t: v * 2.0 ** (-40 - 10 * t)      # down to 2^-70, far below fp16's range
    elif kind == "outlier":
        def fn(v, t):
            v = v.copy()
            v[37 + 500 * t] = 1.0e6 * (1 + t)           # one large value in an ordinary row
            return v
    elif kind == "zero_token":
        fn = lambda v, t: v * 0.0 if t == 1 else v      # a token of zeros between ordinary ones
    else:
        fn = lambda v, t: np.sign(v) * 2.0 ** rng.uniform(-30, 30, size=v.shape)
    run_case(_scaled_x(inp, fn), check_bwd=False)


@pytest.mark.parametrize("M,N,K,r", [
    (1, 64, 64, 8),          # one 64-column block (15 warps without blocks), one tile
    (3, 128, 1088, 24),      # 17 blocks over 16 warps: one warp takes two
    (2, 320, 960, 8),        # 15 blocks: one warp idle
    (4, 2048, 3072, 16),     # several tiles per CTA
    (1, 4096, 4096, 8),      # the decode workload's shape, two tiles per CTA
])
def test_k_ranges_and_tiles(M, N, K, r):
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1400 + M + K), check_bwd=False)


@pytest.mark.parametrize("M,N,K", [
    (4, 11008, 4096),        # five tiles per CTA through two slots
    (1, 8192, 8192),         # four tiles per CTA through one slot
])
def test_tiles_through_a_short_ring(M, N, K):
    """More tiles per CTA than ring slots: the producer refills a slot once all 16 warps
    have released it."""
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=8, seed=1500 + M), check_bwd=False)


@pytest.mark.parametrize("M,N,K,r", [(1, 1024, 4096, 8), (4, 2048, 2048, 64)])
@pytest.mark.parametrize("form", ["single", "fp8"])
def test_other_constant_forms(M, N, K, r, form):
    """Single quantization (fp32 absmax per block) and the FP8-E4M3 second stage."""
    inp = synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1600 + M)
    run_case(inp, check_bwd=False, single=form == "single", fp8=form == "fp8")


@pytest.mark.parametrize("M,N,K,r", [(3, 512, 1024, 64), (2, 256, 512, 256), (4, 640, 2048, 128)])
def test_wide_adapters(M, N, K, r):
    run_case(synth.layer_inputs("tiny", M=M, shape=(N, K), r=r, seed=1700 + r, b_std=1.0), check_bwd=False)


def test_deterministic_and_two_launches():
    """Two calls on the same inputs give identical Y and U; one to four tokens take this
    path (the adapter kernel and the table kernel: two launches), five take the other."""
    inp = synth.layer_inputs("tiny", M=5, shape=(1024, 4096), r=16, seed=1800)
    Wd = torch.from_numpy(inp["W"]).cuda()
    codes, q8, s2 = q.qlora_quantize_nf4_dq(Wd)
    X, A, B = (to_dev_bf16(inp[k]) for k in ("X", "A", "B"))
    for M, launches in ((1, 2), (4, 2), (5, 1)):
        outs = []
        for _ in range(2):
            U = torch.empty(M, 16, dtype=torch.bfloat16, device="cuda")
            n0 = q.qlora_launch_count()
            Y = q.qlora_linear_fwd(codes, q8, s2, 1024, 4096, X[:M].contiguous(), A, B, inp["alpha"], U_save=U)
            torch.cuda.synchronize()
            assert q.qlora_launch_count() - n0 == launches, (M, launches)
            outs.append((Y, U))
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert q.qlora_device_status() == 0


@pytest.mark.parametrize("M,N,K,launches", [
    (1, 4096, 11008, 2),     # the 7B down projection: one 88 KB ring slot, the CTA's tiles through it in turn
    (2, 11008, 4096, 2),     # the 7B gate / up projection: five tiles per CTA
    (3, 4096, 11008, 1),     # three tokens of the down projection exceed the shared memory: tensor-memory path
])
def test_llama7b_shapes(M, N, K, launches):
    """The 7B stack's wide shapes at a few tokens: the table path where its shared memory
    fits, the tensor-memory path where it does not; the same bounds either way."""
    inp = synth.layer_inputs("tiny", M=M, shape=(N, K), r=8, seed=1900 + M)
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(inp["W"]).cuda())
    X, A, B = (to_dev_bf16(inp[k]) for k in ("X", "A", "B"))
    n0 = q.qlora_launch_count()
    q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, inp["alpha"])
    torch.cuda.synchronize()
    assert q.qlora_launch_count() - n0 == launches
    run_case(inp, check_bwd=False)
