"""The C ABI on the host (no GPU): exports, struct layout, validation.

Failure-path tests assert on the returned status and never run a forward pass
(mlxcel issue #974, acceptance criteria: hostile quantisation params fail at
load, each paired with a positive control; Klear PR "Other guards").
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from sparse_moe_ffn_gemv_b200 import build, inputs
from sparse_moe_ffn_gemv_b200 import moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build.build()
    yield


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+(?:const\s+char\s*\*|moe_status)\s*(moe_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) == 16
    assert sorted(M.EXPORTS) == names
    lib = M.lib()
    for n in names:
        assert hasattr(lib, n)
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert set(names) <= exported


def test_struct_layout_matches_the_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe.h"\nint main(void){\n'
                   'printf("%zu %zu %zu %zu %zu\\n", sizeof(moe_config), sizeof(moe_weights),'
                   ' offsetof(moe_config, rms_eps), offsetof(moe_config, routed_scaling_factor),'
                   ' offsetof(moe_weights, latent_norm_w)); printf("%zu\\n", offsetof(moe_weights, gate_up_z));'
                   'return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    assert got == [ctypes.sizeof(M.MoeConfig), ctypes.sizeof(M.MoeWeights),
                   M.MoeConfig.rms_eps.offset, M.MoeConfig.routed_scaling_factor.offset,
                   M.MoeWeights.latent_norm_w.offset, M.MoeWeights.gate_up_z.offset]


def test_enum_values_match_the_header():
    text = open(HEADER).read()
    def val(name):
        return int(re.search(rf"{name}\s*=\s*(\d+)", text).group(1))
    assert val("MOE_SCORING_SIGMOID") == inputs.SCORING["sigmoid"]
    assert val("MOE_SCORING_SOFTMAX_TOPK") == inputs.SCORING["softmax_topk"]
    assert val("MOE_ACT_SWIGLU_CLAMPED") == inputs.ACTIVATION["swiglu_clamped"]
    assert val("MOE_DTYPE_Q4_AFFINE") == inputs.DTYPE["q4"]
    assert val("MOE_DTYPE_MXFP4") == inputs.DTYPE["mxfp4"]
    assert val("MOE_SHARED_BLEND") == inputs.SHARED["blend"]
    for name, code in M.STATUS_CODE.items():
        assert val(name) == code


@pytest.mark.parametrize("spec", list(inputs.WORKLOADS.values()), ids=lambda s: s.name)
def test_every_workload_config_validates(spec):
    assert M.moe_config_validate(M.config_from_spec(spec)) == 0


def _cfg(spec=inputs.KLEAR_BF16, **kw):
    c = M.config_from_spec(spec)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


HOSTILE = [
    ("hidden 0", dict(hidden=0), "MOE_ERR_INVALID_ARGUMENT"),
    ("experts 0", dict(num_experts=0), "MOE_ERR_INVALID_ARGUMENT"),
    ("top_k 0", dict(top_k=0), "MOE_ERR_INVALID_ARGUMENT"),
    ("top_k > E", dict(top_k=257), "MOE_ERR_INVALID_ARGUMENT"),
    ("intermediate 0", dict(intermediate=0), "MOE_ERR_INVALID_ARGUMENT"),
    ("negative hidden", dict(hidden=-2048), "MOE_ERR_INVALID_ARGUMENT"),
    ("bad scoring", dict(scoring=7), "MOE_ERR_INVALID_ARGUMENT"),
    ("bad activation", dict(activation=9), "MOE_ERR_INVALID_ARGUMENT"),
    ("bad shared mode", dict(shared_mode=3), "MOE_ERR_INVALID_ARGUMENT"),
    ("shared width without mode", dict(shared_mode=0), "MOE_ERR_INVALID_ARGUMENT"),
    ("routed scaling 2.5", dict(routed_scaling_factor=2.5), "MOE_ERR_UNSUPPORTED"),
    ("hidden not 16-byte rows", dict(hidden=2044), "MOE_ERR_INVALID_ARGUMENT"),
    ("f32 weights with bf16 acts", dict(weight_format=0), "MOE_ERR_UNSUPPORTED"),
]


@pytest.mark.parametrize("name,fields,expected", HOSTILE, ids=[h[0] for h in HOSTILE])
def test_hostile_config_is_rejected_before_any_launch(name, fields, expected):
    assert M.moe_config_validate(_cfg()) == 0           # positive control first
    assert M.STATUS[M.moe_config_validate(_cfg(**fields))] == expected


QUANT = [("bits 0", dict(bits=0)), ("bits 8", dict(bits=8)), ("group 0", dict(group_size=0)),
         ("group 48", dict(group_size=48)), ("group 256", dict(group_size=256)),
         ("group -64", dict(group_size=-64))]


@pytest.mark.parametrize("name,fields", QUANT, ids=[q[0] for q in QUANT])
def test_hostile_quantisation_params_are_rejected(name, fields):
    assert M.moe_config_validate(_cfg(inputs.KLEAR_Q4)) == 0
    assert M.STATUS[M.moe_config_validate(_cfg(inputs.KLEAR_Q4, **fields))] == "MOE_ERR_INVALID_QUANTIZATION"


def test_mxfp4_needs_blocks_of_32_and_four_bits():
    assert M.moe_config_validate(_cfg(inputs.CLAMPED_MXFP4)) == 0
    for fields in (dict(group_size=64), dict(bits=8)):
        assert M.STATUS[M.moe_config_validate(_cfg(inputs.CLAMPED_MXFP4, **fields))] == \
            "MOE_ERR_INVALID_QUANTIZATION"
    assert M.moe_config_validate(_cfg(inputs.CLAMPED_MXFP4, gate_up_interleaved=1)) == 0  # native layout
    cfg = _cfg(inputs.CLAMPED_MXFP4)
    w = _fake_weights(inputs.CLAMPED_MXFP4)
    w.gate_z = w.up_z = w.down_z = w.gate_up_s = w.gate_up_z = None  # no affine biases; split planes
    assert M.moe_weights_validate(cfg, w) == 0
    w.down_s = None                                  # but every plane needs its scales
    assert M.STATUS[M.moe_weights_validate(cfg, w)] == "MOE_ERR_MISSING_TENSOR"


@pytest.mark.parametrize("fmt", ["mxfp4", "q4"])
def test_interleaved_4bit_plane_needs_its_own_companions(fmt):
    """With one gate_up plane (libmir-metal ExpertLayout::Native) the scales (and Q4 biases)
    come from gate_up_s / gate_up_z; the split planes' companions are not consulted."""
    spec = inputs.CLAMPED_MXFP4.replace(gate_up_interleaved=True, weight_format=fmt)
    cfg = _cfg(spec)
    w = _fake_weights(spec)
    w.gate_s = w.gate_z = w.up_s = w.up_z = None
    assert M.moe_weights_validate(cfg, w) == 0
    for f in (["gate_up_s", "gate_up_z"] if fmt == "q4" else ["gate_up_s"]):
        w2 = _fake_weights(spec)
        setattr(w2, f, None)
        assert M.STATUS[M.moe_weights_validate(cfg, w2)] == "MOE_ERR_MISSING_TENSOR", f
    w3 = _fake_weights(spec)
    w3.gate_up_s = 1 << 21 | 8                       # misaligned companion plane
    assert M.STATUS[M.moe_weights_validate(cfg, w3)] == "MOE_ERR_INVALID_ARGUMENT"


def test_4bit_dense_planes_are_validated_before_any_launch():
    """4-bit router / shared / latent planes (mlxcel issue #974, the Jamba study): accepted with
    bf16 activations and a group that divides every width; hostile parameters are refused,
    each beside a positive control."""
    from tiny_specs import DENSE_Q4, DENSE_Q4_BLEND
    for spec in (DENSE_Q4, DENSE_Q4_BLEND):
        assert M.moe_config_validate(M.config_from_spec(spec)) == 0
    bad_group = M.config_from_spec(DENSE_Q4)
    bad_group.dense_group_size = 48
    assert M.STATUS[M.moe_config_validate(bad_group)] == "MOE_ERR_INVALID_QUANTIZATION"
    assert M.STATUS[M.moe_config_validate(M.config_from_spec(DENSE_Q4.replace(dense_group_size=128)))] == \
        "MOE_ERR_INVALID_QUANTIZATION"                       # 128 does not divide hidden 64
    bad_fmt = M.config_from_spec(DENSE_Q4)
    bad_fmt.dense_format = 3                                 # MXFP4 dense planes: not a dense format here
    assert M.STATUS[M.moe_config_validate(bad_fmt)] == "MOE_ERR_INVALID_ARGUMENT"
    f32 = M.config_from_spec(inputs.TINY_F32)
    f32.dense_format = 2
    assert M.STATUS[M.moe_config_validate(f32)] == "MOE_ERR_UNSUPPORTED"
    with pytest.raises(ValueError, match="dense_format"):
        M.config_from_spec(DENSE_Q4.replace(dense_format="mxfp4"))


def test_4bit_dense_planes_need_their_scales_and_biases():
    from tiny_specs import DENSE_Q4
    cfg = M.config_from_spec(DENSE_Q4)
    w = inputs.make_weights(DENSE_Q4, threads=2)
    ws = M.weights_struct(w)
    assert M.moe_weights_validate(cfg, ws) == 0
    for f in ("router_s", "shared_down_z", "latent_up_s"):
        broken = M.weights_struct({k: v for k, v in w.items() if k != f})
        assert M.STATUS[M.moe_weights_validate(cfg, broken)] == "MOE_ERR_MISSING_TENSOR", f


def test_group_must_divide_the_widths():
    spec = inputs.KLEAR_Q4.replace(intermediate=800)      # 800 % 64 != 0
    assert M.STATUS[M.moe_config_validate(M.config_from_spec(spec))] == "MOE_ERR_INVALID_QUANTIZATION"
    assert M.moe_config_validate(M.config_from_spec(spec.replace(group_size=32))) == 0


def test_nonfinite_eps_and_limit_are_rejected():
    assert M.moe_config_validate(_cfg(inputs.LATENT_BF16)) == 0
    for eps in (0.0, -1e-6, float("inf"), float("nan")):
        assert M.moe_config_validate(_cfg(inputs.LATENT_BF16, rms_eps=eps)) == 1
    assert M.moe_config_validate(_cfg(inputs.CLAMPED_BF16)) == 0
    for lim in (0.0, float("nan")):
        assert M.moe_config_validate(_cfg(inputs.CLAMPED_BF16, swiglu_limit=lim)) == 1


def _fake_weights(spec, align=16):
    """Host addresses stand in for device pointers: validation never dereferences them."""
    w = M.MoeWeights()
    base = 1 << 20
    for i, f in enumerate(M.WEIGHT_FIELDS):
        setattr(w, f, base + i * 4096 + (0 if align == 16 else 8))
    return w


def test_missing_coefficient_head_is_rejected():
    cfg = _cfg()
    w = _fake_weights(inputs.KLEAR_BF16)
    assert M.moe_weights_validate(cfg, w) == 0
    w.coef_w = None
    assert M.STATUS[M.moe_weights_validate(cfg, w)] == "MOE_ERR_MISSING_TENSOR"


def test_missing_q4_companions_and_misaligned_pointers_are_rejected():
    cfg = _cfg(inputs.KLEAR_Q4)
    w = _fake_weights(inputs.KLEAR_Q4)
    assert M.moe_weights_validate(cfg, w) == 0
    w.down_z = None
    assert M.STATUS[M.moe_weights_validate(cfg, w)] == "MOE_ERR_MISSING_TENSOR"
    assert M.STATUS[M.moe_weights_validate(cfg, _fake_weights(inputs.KLEAR_Q4, align=8))] == \
        "MOE_ERR_INVALID_ARGUMENT"


def test_workspace_size_grows_with_tokens_and_rejects_overflow():
    cfg = _cfg()
    sizes = [M.moe_workspace_size(cfg, T) for T in (0, 1, 8, 64, 4096)]
    assert sizes == sorted(sizes) and sizes[-1] > sizes[1] > 0
    with pytest.raises(M.MoeError) as e:
        M.moe_workspace_size(cfg, 1 << 40)
    assert e.value.name == "MOE_ERR_SHAPE_OVERFLOW"
    with pytest.raises(M.MoeError):
        M.moe_workspace_size(cfg, -1)


def test_zero_tokens_is_a_no_op_and_errors_precede_launches():
    lib = M.lib()
    cfg = _cfg()
    w = _fake_weights(inputs.KLEAR_BF16)
    # T == 0: MOE_OK, nothing launched (this host has no GPU at all)
    assert lib.moe_block_forward(ctypes.byref(cfg), ctypes.byref(w), None, 0, None, None, 0, None) == 0
    # T > 0 with a workspace that is too small: rejected on the host
    ws = ctypes.c_void_p(1 << 24)
    assert M.STATUS[lib.moe_block_forward(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(1 << 22), 4,
                                          ctypes.c_void_p(1 << 23), ws, 16, None)] == \
        "MOE_ERR_WORKSPACE_TOO_SMALL"
    bad = _cfg(top_k=0)
    assert M.STATUS[lib.moe_block_forward(ctypes.byref(bad), ctypes.byref(w), ctypes.c_void_p(1 << 22), 4,
                                          ctypes.c_void_p(1 << 23), ws, 1 << 30, None)] == \
        "MOE_ERR_INVALID_ARGUMENT"
    # a NULL output pointer is rejected too
    assert M.STATUS[lib.moe_block_forward(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(1 << 22), 4,
                                          None, ws, 1 << 30, None)] == "MOE_ERR_INVALID_ARGUMENT"


def test_noalloc_permutation_rejects_sizes_beyond_its_fixed_scratch():
    """The allocation-free permutation checks its limits on the host, before any launch."""
    lib = M.lib()
    cfg = _cfg()                      # top_k 8: 8193 tokens are 65,544 slots > 65,536
    p = ctypes.c_void_p(1 << 22)
    assert M.STATUS[lib.moe_permute_noalloc(ctypes.byref(cfg), p, 8193, p, p, p, None, None)] == \
        "MOE_ERR_SHAPE_OVERFLOW"
    assert lib.moe_permute_noalloc(ctypes.byref(cfg), p, 0, p, p, p, None, None) == 0
    assert M.STATUS[lib.moe_permute_noalloc(ctypes.byref(_cfg(top_k=0)), p, 4, p, p, p, None, None)] == \
        "MOE_ERR_INVALID_ARGUMENT"


def test_selftest_rejects_bad_arguments_before_any_launch():
    lib = M.lib()
    for fn in (lib.moe_selftest_bounded_wait, lib.moe_selftest_grid_wait):
        assert M.STATUS[fn(None, 1000, None)] == "MOE_ERR_INVALID_ARGUMENT"
        for ns in (0, -5, 2_000_000_000):
            assert M.STATUS[fn(ctypes.c_void_p(1 << 20), ns, None)] == "MOE_ERR_INVALID_ARGUMENT"


def test_status_strings():
    lib = M.lib()
    for code in M.STATUS:
        assert lib.moe_status_string(code)
    assert lib.moe_status_string(99) == b"unknown status"


def test_product_path_has_no_fallback(monkeypatch):
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "LIB_PATH", "/nonexistent/libmoe_b200.so")
    with pytest.raises(RuntimeError):
        M.lib()
