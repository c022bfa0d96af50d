"""The bench's algorithmic-traffic and FLOP model against hand arithmetic, on the CPU.

The roofline fraction the bench reports is algorithmic bytes (or FLOPs) per launch
divided by the measured launch time; these checks pin that numerator for the
workloads' layers to numbers worked out by hand here (bf16, s = 2 bytes)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dynamic_short_convolutions_b200 import workloads as W  # noqa: E402

C2 = W.CONFIGS["c2_qkv_150m_lowrank"]        # N = 8 x 2048 = 16384, d 768, C 2304, K 3, r 32
C3 = W.CONFIGS["c3_qkv_2b_headwise_gqa"]     # N = 16384, d 2048, C 3072, K 4, 24 heads of 128


def test_lowrank_backward_bytes_per_launch():
    # reads g, u, writes du: 3 * 16384 * 2304 * 2 = 226 492 416
    # reads z: 16384 * 32 * 2 = 1 048 576; reads B: 32 * 2304 * 3 * 2 = 442 368
    assert bench.kernel_bytes("tc_lowrank_bwd", C2, C2.layers[0]) == 227_983_360


def test_lowrank_forward_and_generator_bytes_per_launch():
    # forward: u, y (2 * 16384 * 2304 * 2 = 150 994 944) + z (1 048 576) + B (442 368)
    assert bench.kernel_bytes("tc_lowrank_fwd", C2, C2.layers[0]) == 152_485_888
    # generator: h (16384 * 768 * 2 = 25 165 824) + A (768 * 32 * 2 = 49 152) + z (1 048 576)
    assert bench.kernel_bytes("tc_gen", C2, C2.layers[0]) == 26_263_552


def test_headwise_conv_bytes_per_launch():
    # backward: g, u, du (3 * 16384 * 3072 * 2 = 301 989 888) + filters and dwh (16384 * 96 * 2 each)
    assert bench.kernel_bytes("tc_headwise_bwd", C3, C3.layers[0]) == 301_989_888 + 2 * 16384 * 96 * 2
    # forward: u, y (2 * 16384 * 3072 * 2 = 201 326 592) + filters (16384 * 96 * 2 = 3 145 728)
    assert bench.kernel_bytes("tc_headwise_fwd", C3, C3.layers[0]) == 204_472_320


def test_layer_bytes_and_flops_of_the_150m_qkv_layer():
    # per token: fwd u, y, h = 2 (2 * 2304 + 768) = 10 752; bwd g, u, du, h = 2 (3 * 2304 + 768) = 15 360;
    # dh = 1 536; z written and read = 128  ->  27 776 bytes, x 16384 tokens = 455 081 984
    # parameters: A and B read in both passes 2 * 2 * (24 576 + 221 184) = 983 040, dA and dB in fp32 983 040
    assert bench.layer_bytes(C2, C2.layers[0]) == 455_081_984 + 983_040 + 983_040
    # per token 8 r C K (w, w again, dz, dB) + 6 d r (z, dA, dh) = 1 769 472 + 147 456 = 1 916 928 FLOPs
    assert bench.layer_flops(C2, C2.layers[0]) == 16384 * 1_916_928


def test_every_library_kernel_has_a_byte_model():
    for name in ("tc_gen", "tc_lowrank_fwd", "tc_lowrank_bwd", "tc_gen_bwd", "simt_conv_fwd", "simt_conv_bwd"):
        assert bench.kernel_bytes(name, C2, C2.layers[0]) > 0
    for name in ("tc_headwise_fwd", "tc_headwise_bwd"):
        assert bench.kernel_bytes(name, C3, C3.layers[0]) > 0
