"""bench.py's algorithmic byte and flop counts, checked by hand on the workload shapes.

The roofline fractions divide these counts by measured times, so a wrong count (e.g. a
4-bit plane counted at bf16 width) inflates every fraction reported for that format.
"""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from sparse_moe_ffn_gemv_b200 import inputs  # noqa: E402


def test_expert_bytes_per_format():
    # Klear bf16: gate, up [768, 2048] and down [2048, 768], 2 bytes each
    assert bench.expert_bytes(inputs.KLEAR_BF16) == 3 * 768 * 2048 * 2
    # Klear 4-bit affine, group 64: half a byte per weight + bf16 scale and bias per group
    assert bench.expert_bytes(inputs.KLEAR_Q4) == 3 * 768 * 2048 // 2 + 3 * 768 * (2048 // 64) * 4
    # clamped bf16: three 2880 x 2880 planes + the gate/up and down biases
    assert bench.expert_bytes(inputs.CLAMPED_BF16) == 3 * 2880 * 2880 * 2 + 3 * 2880 * 2
    # clamped MXFP4 (split or native): half a byte per weight + one scale byte per 32 + biases
    for spec in (inputs.CLAMPED_MXFP4, inputs.CLAMPED_MXFP4_NATIVE):
        assert bench.expert_bytes(spec) == 3 * 2880 * 2880 // 2 + 3 * 2880 * 90 + 3 * 2880 * 2
    # per-expert megabytes of the workload table: 9.44 (Klear), 2.65 (4-bit), 49.8 (clamped)
    assert round(bench.expert_bytes(inputs.KLEAR_BF16) / 1e6, 2) == 9.44
    assert round(bench.expert_bytes(inputs.KLEAR_Q4) / 1e6, 2) == 2.65
    assert round(bench.expert_bytes(inputs.CLAMPED_BF16) / 1e6, 1) == 49.8


def test_block_flops_counts_router_experts_and_shared():
    s = inputs.KLEAR_BF16
    T = 4096
    want = 2 * T * 256 * 2048 + 2 * T * 8 * 3 * 768 * 2048 + 2 * T * 3 * 768 * 2048
    assert bench.block_flops(s, T) == want
