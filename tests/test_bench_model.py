"""The algorithmic work behind bench.py's roofline numbers, checked on CPU.

The achieved figures the bench reports are these bytes or FLOPs per launch
divided by measured launch times, so the model is pinned here to values
worked out by hand from the block formats and the layer shapes.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

H, I, E, K = 4096, 2048, 256, 8
IQ2_MATRIX = I * H // 256 * 66      # 2,162,688 bytes of IQ2 blocks per gate or up matrix
Q2_MATRIX = H * I // 256 * 84       # 2,752,512 bytes of Q2 blocks per down matrix


def test_block_matrix_sizes():
    assert IQ2_MATRIX == 2_162_688 and Q2_MATRIX == 2_752_512
    assert 2 * IQ2_MATRIX + Q2_MATRIX == 7_077_888          # one routed expert


def test_decode_bytes_one_token():
    ab = bench.algorithmic_bytes(bench.WORKLOADS["decode"], 8)
    # 8 experts' blocks + the bf16 shared expert + x + h written and read (9 rows of I values, 4 bytes) + y
    assert ab["k_moe_decode"] == 8 * 7_077_888 + 3 * I * H * 2 + H * 4 + 2 * 9 * I * 4 + 9 * H * 4 == 107_266_048
    # router rows + 8 routed experts + the whole shared expert
    assert ab["layer"] == E * H * 4 + 8 * 7_077_888 + 3 * I * H * 2 == 111_149_056
    assert ab["routed"] == 8 * 7_077_888


def test_decode_bytes_scale_with_distinct_experts():
    w = bench.WORKLOADS["decode2"]
    a, b = bench.algorithmic_bytes(w, 8), bench.algorithmic_bytes(w, 16)
    assert b["routed"] - a["routed"] == 8 * 7_077_888
    assert b["k_moe_decode"] - a["k_moe_decode"] == 8 * 7_077_888


def test_prefill_flops_and_bytes():
    w = bench.WORKLOADS["prefill11709"]
    fl = bench.algorithmic_flops(w)
    slots = 11_709 * K
    assert fl["k_moe_gemm<gate_up>"] == 2 * slots * H * 2 * I == 3_143_110_754_304
    assert fl["k_moe_gemm<down>"] == fl["k_moe_gemm<gate_up>"] // 2
    assert fl["k_moe_gemm<shared_gate_up>"] == 2 * 11_709 * H * 2 * I
    ab = bench.algorithmic_bytes(w, 256)
    # every expert's gate and up blocks once, the permuted bf16 activations in, h out in bf16
    assert ab["k_moe_gemm<gate_up>"] == 256 * 2 * IQ2_MATRIX + slots * H * 2 + slots * I * 2


def test_secondary_peaks_are_the_nominal_figures():
    assert bench.NOMINAL["hbm_gbs"] == pytest.approx(7700.0)
    assert bench.NOMINAL["bf16_tflops"] == pytest.approx(2250.0)
