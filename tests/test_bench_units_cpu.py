"""The bench's algorithmic units against closed forms that the pages and the method fix.

The roofline fractions divide these numbers by measured times, so each is pinned here to an
independent statement of the same quantity:

* decode bytes: the packed weight at 4 bit/param plus the double-quantized constants at
  8/64 + 32/(64 * 256) bit/param ("QLoRAの理論と実装" §5-2, memory arithmetic with DQ);
* quantize bytes: the fp32 input (32 bit/param) plus that output;
* training FLOP: two dense products of 2MNK each for Y and dX, and the adapter's
  four skinny products of the forward and backward (U, U B^T, V, V A) plus dA and dB.
"""
import os
import sys
from fractions import Fraction

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def bits_per_param_dq():
    return Fraction(4) + Fraction(8, 64) + Fraction(32, 64 * 256)


def test_decode_bytes_are_the_dq_bits_per_param():
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008), (8192, 8192), (22016, 8192)):
        assert Fraction(bench.decode_weight_bytes(N, K)) == N * K * bits_per_param_dq() / 8, (N, K)
    assert bench.decode_weight_bytes(4096, 4096) == 8_388_608 + 262_144 + 4_096


def test_quantize_bytes_add_the_fp32_input():
    for N, K in ((4096, 4096), (8192, 22016)):
        assert Fraction(bench.quant_bytes(N, K)) == N * K * (32 + bits_per_param_dq()) / 8
    assert bench.quant_bytes(4096, 4096) == 75_763_712


def test_training_flop():
    M = N = K = 4096
    r = 64
    main = 2 * (2 * M * N * K)                       # Y = X W^T and dX = dY W
    adapter = 2 * M * K * r + 2 * M * r * N          # U = X A^T, then U B^T
    adapter += 2 * M * N * r + 2 * M * r * K         # V = dY B, then V A
    adapter += 2 * r * M * K + 2 * N * M * r         # dA = V^T X, dB = dY^T U
    assert bench.step_flops(M, N, K, r) == main + adapter == 287_762_808_832
    assert bench.kernel_flops("fwd_fused", M, N, K, r) == 2 * M * N * K + 2 * M * N * r == 139_586_437_120
    assert bench.kernel_flops("dx_fused", M, N, K, r) == 2 * M * N * K + 2 * M * K * r
