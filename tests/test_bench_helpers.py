"""Host-side helpers of bench.py, without a GPU: the algorithmic byte counts
that every GB/s figure divides by, and the rule that a committed ncu traffic
figure is used only while the profiled kernel source is unchanged."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bitlinear_absmean_ternary_b200 import synth  # noqa: E402


def test_linear_bytes_of_the_decode_workload():
    up, down = synth.WORKLOADS["decode_m1_2p5b_ffn"]
    b = bench.linear_bytes(up)
    # bf16 x in, x_q + a + rowsum out
    assert b["quant"] == 2 * 2560 + 2560 + 8
    # packed W (2 bits), x_q, a + rowsum, gamma, bf16 y
    assert b["product"] == 6912 * 2560 // 4 + 2560 + 8 + 4 + 2 * 6912
    assert b["x_in"] == 2 * 2560 and b["y_out"] == 2 * 6912
    bd = bench.linear_bytes(down)
    assert bd["product"] == 2560 * 6912 // 4 + 6912 + 8 + 4 + 2 * 2560


def test_linear_bytes_counts_the_norm_gain():
    lin = synth.WORKLOADS["decode_m64_2p5b_block"][0]
    assert lin.norm
    b = bench.linear_bytes(lin)
    assert b["quant"] == 64 * 2560 * 2 + 2560 * 2 + 64 * 2560 + 8 * 64


def test_profiled_traffic_requires_a_matching_source_hash(tmp_path):
    h = bench.kernel_source_hash(["gemv.cuh", "quant.cuh", "ptx.cuh"])
    assert len(h) == 16 and h != bench.kernel_source_hash(["gemm.cuh", "ptx.cuh"])
    f = tmp_path / "summary.md"
    f.write_text(f"text\ntraffic_bytes_per_launch: 123456\nkernel_source_hash: {h}\n")
    assert bench.profiled_traffic(str(f), h) == 123456.0
    assert bench.profiled_traffic(str(f), "0" * 16) is None
    assert bench.profiled_traffic(str(tmp_path / "missing.md"), h) is None
