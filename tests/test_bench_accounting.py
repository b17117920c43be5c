"""bench.py's algorithmic byte and flop counts, checked by hand on the workload shapes.

The roofline fractions divide these counts by measured times, so a wrong count (e.g. a
4-bit plane counted at bf16 width) inflates every fraction reported for that format.
"""
import os
import sys
import pytest

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


def test_l2_flush_between_timed_steps_only_where_the_weights_could_stay_in_l2():
    # Klear bf16 prefill: 256 experts x 9.44 MB, far above 2 x 126 MB -> no flush needed
    assert not bench.needs_l2_flush(inputs.KLEAR_BF16, 4096)
    assert not bench.needs_l2_flush(inputs.KLEAR_BF16, 64)      # up to 256 experts activated
    # one token: 8 experts (76 MB bf16, 21 MB 4-bit) plus the dense weights fit in L2 twice
    assert bench.needs_l2_flush(inputs.KLEAR_BF16, 1)
    assert bench.needs_l2_flush(inputs.KLEAR_Q4, 1)
    assert bench.needs_l2_flush(inputs.KLEAR_Q4, 8)             # 64 x 2.65 MB = 170 MB < 252 MB
    assert not bench.needs_l2_flush(inputs.KLEAR_Q4, 32)        # up to 256 x 2.65 MB = 679 MB
    for spec, T in ((inputs.KLEAR_Q4, 1), (inputs.KLEAR_BF16, 4096)):
        cfg = bench.workload_config(spec, T, 1)
        assert cfg["l2"].startswith("L2 flushed" if bench.needs_l2_flush(spec, T) else "activated weights larger")


def test_expert_launch_bytes_add_up_to_the_expert_planes():
    """The gate/up and down launches read the routed planes once: their weight bytes
    sum to the distinct experts' bytes plus the shared planes."""
    s = inputs.KLEAR_BF16
    T, nd = 4096, 216
    r = bench.kernel_roles(s, T, nd)
    H, k, I, Is = s.hidden, s.top_k, s.intermediate, s.shared_intermediate
    io_gu = T * H * 2 + T * H * 2 + T * k * I * 2 + T * Is * 2       # u, x in; h, hs out
    io_dn = T * k * I * 2 + T * Is * 2 + T * H * 4 + T * H * 4       # h, hs in; sums out
    assert r["gate/up"]["bytes"] - io_gu + r["down"]["bytes"] - io_dn == nd * bench.expert_bytes(s) + 3 * Is * H * 2
    assert r["gate/up"]["flops"] + r["down"]["flops"] + 2 * T * 256 * 2048 == bench.block_flops(s, T)


def test_kernel_names_from_mangled_symbols():
    n = bench.short_kernel_name
    assert n("_ZN3moe12_GLOBAL__N_114tc_gemm_kernelILb1ELi128ELi4ELb0EEEvNS_8TcParamsE") == "tc_gemm_kernel<1,128,4,0>"
    assert n("_ZN3moe12_GLOBAL__N_118gateup_gemv_kernelILi1EEEvNS_10GateUpArgsE") == "gateup_gemv_kernel<1>"
    assert n("_ZN3moe12_GLOBAL__N_111topk_kernelENS_8TopkArgsE") == "topk_kernel"
    table = [("topk_kernel", 1.0), ("tc_gemm_kernel<1,128,4,0>", 3.0), ("tc_gemm_kernel<0,128,4,0>", 2.0)]
    assert bench.label_expert_launches(table) == (1, 2)


def test_headline_is_the_largest_single_gpu_workload():
    args = bench.parse([])
    assert (args.workload, args.tokens) == ("latent_bf16", 8192)
    big = max(bench.PREFILL, key=lambda w: bench.block_flops(inputs.WORKLOADS[w], bench.PREFILL[w]))
    assert big == "latent_bf16"


def test_dense_bytes_count_4bit_dense_planes_at_their_width():
    s = inputs.KLEAR_Q4_DENSE
    H, E, Is, g = s.hidden, s.num_experts, s.shared_intermediate, s.dense_group_size
    q4 = lambda r, c: r * c // 2 + r * (c // g) * 4
    assert bench.dense_bytes(s) == q4(E, H) + E * 4 + 2 * H * 2 + 3 * q4(Is, H)
    assert bench.dense_bytes(s) < bench.dense_bytes(inputs.KLEAR_Q4) / 3


def test_smaller_copy_of_a_workload_keeps_every_other_field():
    import bench
    a = bench.parse(["--workload", "latent_bf16", "--tokens", "8192", "--experts", "32"])
    s = bench.workload_spec(a)
    full = bench.inputs.WORKLOADS["latent_bf16"]
    assert s.num_experts == 32 and s.name == "latent_bf16_e32"
    assert (s.hidden, s.latent_dim, s.top_k, s.intermediate, s.config_id) == \
        (full.hidden, full.latent_dim, full.top_k, full.intermediate, full.config_id)
    assert bench.workload_spec(bench.parse(["--workload", "klear_bf16"])) is bench.inputs.WORKLOADS["klear_bf16"]
    with pytest.raises(SystemExit):
        bench.workload_spec(bench.parse(["--workload", "klear_bf16", "--experts", "4"]))


def test_kernel_source_hash_ignores_comments_but_not_code():
    import bench
    a = "int f(int x) { return x + 1; } // add one\n"
    assert bench.code_of(a) == bench.code_of("/* doc */\nint f(int x) { return x + 1; }\n\n")
    assert bench.code_of(a) != bench.code_of("int f(int x) { return x + 2; }\n")
