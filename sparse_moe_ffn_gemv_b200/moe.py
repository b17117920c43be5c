"""Thin Python binding of libmoe_b200.so (include/moe.h).

Argument marshalling only: every step of the block runs in the library's CUDA
kernels. PyTorch supplies device memory and streams. There is no fallback: if
the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

from . import inputs

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")

WEIGHT_FIELDS = [
    "router_w", "router_b", "selection_bias", "coef_w", "coef_b",
    "gate_w", "up_w", "gate_up_w", "gate_b", "up_b", "gate_up_b", "down_w", "down_b",
    "gate_s", "gate_z", "up_s", "up_z", "down_s", "down_z",
    "shared_gate_w", "shared_up_w", "shared_down_w",
    "latent_down_w", "latent_up_w", "latent_norm_w",
    "gate_up_s", "gate_up_z",
    "router_s", "router_z", "shared_gate_s", "shared_gate_z", "shared_up_s", "shared_up_z",
    "shared_down_s", "shared_down_z", "latent_down_s", "latent_down_z", "latent_up_s", "latent_up_z",
]

# The entry points include/moe.h declares.
EXPORTS = [
    "moe_config_validate", "moe_weights_validate", "moe_workspace_size", "moe_route",
    "moe_permute", "moe_grouped_ffn", "moe_grouped_ffn_experts", "moe_latent_down", "moe_combine", "moe_block_forward",
    "moe_read_device_status", "moe_clear_device_status", "moe_status_string",
    "moe_permute_noalloc", "moe_selftest_bounded_wait", "moe_selftest_grid_wait",
]

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_SHAPE_OVERFLOW",
          3: "MOE_ERR_INVALID_QUANTIZATION", 4: "MOE_ERR_MISSING_TENSOR", 5: "MOE_ERR_UNSUPPORTED",
          6: "MOE_ERR_CUDA", 7: "MOE_ERR_DEVICE_CHECK", 8: "MOE_ERR_DEVICE_TIMEOUT",
          9: "MOE_ERR_WORKSPACE_TOO_SMALL"}
STATUS_CODE = {v: k for k, v in STATUS.items()}


class MoeConfig(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("intermediate", ctypes.c_int32), ("scoring", ctypes.c_int32),
        ("norm_topk_prob", ctypes.c_int32), ("routed_scaling_factor", ctypes.c_float),
        ("activation", ctypes.c_int32), ("swiglu_limit", ctypes.c_float),
        ("swiglu_alpha", ctypes.c_float), ("gate_up_interleaved", ctypes.c_int32),
        ("has_expert_bias", ctypes.c_int32), ("has_router_bias", ctypes.c_int32),
        ("has_selection_bias", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
        ("weight_format", ctypes.c_int32), ("group_size", ctypes.c_int32), ("bits", ctypes.c_int32),
        ("shared_mode", ctypes.c_int32), ("shared_intermediate", ctypes.c_int32),
        ("latent_dim", ctypes.c_int32), ("latent_use_norm", ctypes.c_int32),
        ("rms_eps", ctypes.c_float), ("dense_format", ctypes.c_int32), ("dense_group_size", ctypes.c_int32),
    ]


class MoeWeights(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in WEIGHT_FIELDS]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name} ({_status_string(status)})")


_lib = None


def lib():
    """The loaded CUDA library (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with sparse_moe_ffn_gemv_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        cfgp, wp = ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights)
        sig = {
            "moe_config_validate": [cfgp],
            "moe_weights_validate": [cfgp, wp],
            "moe_workspace_size": [cfgp, i64, ctypes.POINTER(sz)],
            "moe_route": [cfgp, wp, vp, i64, vp, vp, vp, vp, sz, vp],
            "moe_permute": [cfgp, vp, i64, vp, vp, vp, vp, sz, vp],
            "moe_grouped_ffn": [cfgp, wp, vp, i64, vp, vp, vp, vp, vp, sz, vp],
            "moe_grouped_ffn_experts": [cfgp, wp, vp, i64, vp, vp, vp, ctypes.c_int32, ctypes.c_int32, vp, vp, sz,
                                        vp],
            "moe_latent_down": [cfgp, wp, vp, i64, vp, vp, sz, vp],
            "moe_combine": [cfgp, wp, vp, vp, vp, i64, vp, vp, sz, vp],
            "moe_block_forward": [cfgp, wp, vp, i64, vp, vp, sz, vp],
            "moe_read_device_status": [vp, vp],
            "moe_clear_device_status": [vp, vp],
            "moe_permute_noalloc": [cfgp, vp, i64, vp, vp, vp, vp, vp],
            "moe_selftest_bounded_wait": [vp, i64, vp],
            "moe_selftest_grid_wait": [vp, i64, vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().moe_status_string(status).decode()
    except Exception:  # the library itself may be what is missing
        return STATUS.get(status, "?")


def _check(status: int, where: str):
    if status != 0:
        raise MoeError(status, where)


def config_from_spec(spec) -> MoeConfig:
    dense = getattr(spec, "dense_format", "act")
    if dense not in ("act", "q4"):
        raise ValueError(f"dense_format {dense!r}")
    return MoeConfig(
        hidden=spec.hidden, num_experts=spec.num_experts, top_k=spec.top_k,
        intermediate=spec.intermediate, scoring=inputs.SCORING[spec.scoring],
        norm_topk_prob=int(spec.norm_topk_prob),
        routed_scaling_factor=float(spec.routed_scaling_factor),
        activation=inputs.ACTIVATION[spec.activation], swiglu_limit=float(spec.swiglu_limit),
        swiglu_alpha=float(spec.swiglu_alpha), gate_up_interleaved=int(spec.gate_up_interleaved),
        has_expert_bias=int(spec.has_expert_bias), has_router_bias=int(spec.has_router_bias),
        has_selection_bias=int(spec.has_selection_bias), act_dtype=inputs.DTYPE[spec.act_dtype],
        weight_format=inputs.DTYPE[spec.weight_format], group_size=spec.group_size,
        bits=spec.bits, shared_mode=inputs.SHARED[spec.shared_mode],
        shared_intermediate=spec.shared_intermediate, latent_dim=spec.latent_dim,
        latent_use_norm=int(spec.latent_use_norm), rms_eps=float(spec.rms_eps),
        dense_format=inputs.DTYPE["q4"] if dense == "q4" else 0, dense_group_size=int(spec.dense_group_size))


def weights_struct(dev: Dict[str, torch.Tensor]) -> MoeWeights:
    w = MoeWeights()
    for f in WEIGHT_FIELDS:
        t = dev.get(f)
        if t is not None:
            setattr(w, f, t.data_ptr())
    return w


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------- same-named calls
def moe_config_validate(cfg: MoeConfig) -> int:
    return lib().moe_config_validate(ctypes.byref(cfg))


def moe_weights_validate(cfg: MoeConfig, w: MoeWeights) -> int:
    return lib().moe_weights_validate(ctypes.byref(cfg), ctypes.byref(w))


def moe_workspace_size(cfg: MoeConfig, max_tokens: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(cfg), int(max_tokens), ctypes.byref(out)),
           "moe_workspace_size")
    return out.value


def moe_route(cfg, w, x, T, topk_idx, topk_w, coef, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(cfg), ctypes.byref(w), _p(x), int(T), _p(topk_idx),
                           _p(topk_w), _p(coef), _p(ws), ws.numel(), _stream(stream)), "moe_route")


def moe_permute(cfg, topk_idx, T, expert_offsets, sorted_slot, slot_pos, ws, stream=None):
    _check(lib().moe_permute(ctypes.byref(cfg), _p(topk_idx), int(T), _p(expert_offsets),
                             _p(sorted_slot), _p(slot_pos), _p(ws), ws.numel(), _stream(stream)),
           "moe_permute")


def moe_grouped_ffn(cfg, w, u, T, expert_offsets, sorted_slot, topk_w, y_acc, ws, stream=None):
    _check(lib().moe_grouped_ffn(ctypes.byref(cfg), ctypes.byref(w), _p(u), int(T),
                                 _p(expert_offsets), _p(sorted_slot), _p(topk_w), _p(y_acc),
                                 _p(ws), ws.numel(), _stream(stream)), "moe_grouped_ffn")


def moe_grouped_ffn_experts(cfg, w, u, T, expert_offsets, sorted_slot, topk_w, expert_begin, expert_end,
                            y_acc, ws, stream=None):
    """Routed experts [expert_begin, expert_end) only; w's routed planes hold just those."""
    _check(lib().moe_grouped_ffn_experts(ctypes.byref(cfg), ctypes.byref(w), _p(u), int(T),
                                         _p(expert_offsets), _p(sorted_slot), _p(topk_w), int(expert_begin),
                                         int(expert_end), _p(y_acc), _p(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn_experts")


def moe_latent_down(cfg, w, x, T, z, ws, stream=None):
    _check(lib().moe_latent_down(ctypes.byref(cfg), ctypes.byref(w), _p(x), int(T), _p(z),
                                 _p(ws), ws.numel(), _stream(stream)), "moe_latent_down")


def moe_combine(cfg, w, y_acc, x, coef, T, y, ws, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), ctypes.byref(w), _p(y_acc), _p(x), _p(coef),
                             int(T), _p(y), _p(ws), ws.numel(), _stream(stream)), "moe_combine")


def moe_block_forward(cfg, w, x, T, y, ws, stream=None):
    _check(lib().moe_block_forward(ctypes.byref(cfg), ctypes.byref(w), _p(x), int(T), _p(y),
                                   _p(ws), ws.numel(), _stream(stream)), "moe_block_forward")


def moe_permute_noalloc(cfg, topk_idx, T, expert_offsets, sorted_slot, slot_pos, device_status=None,
                        stream=None):
    """moe_permute without a workspace: the library keeps the scratch in a fixed device
    array (for callers that cannot allocate device memory where they route tokens)."""
    _check(lib().moe_permute_noalloc(ctypes.byref(cfg), _p(topk_idx), int(T), _p(expert_offsets),
                                     _p(sorted_slot), _p(slot_pos), _p(device_status), _stream(stream)),
           "moe_permute_noalloc")


def moe_selftest_bounded_wait(ws, timeout_ns: int, stream=None):
    """Run the bounded-wait self test: records MOE_ERR_DEVICE_TIMEOUT in ws's status word."""
    _check(lib().moe_selftest_bounded_wait(_p(ws), int(timeout_ns), _stream(stream)), "moe_selftest_bounded_wait")


def moe_selftest_grid_wait(ws, timeout_ns: int, stream=None):
    """Run the grid-barrier self test: records MOE_ERR_DEVICE_TIMEOUT in ws's status word."""
    _check(lib().moe_selftest_grid_wait(_p(ws), int(timeout_ns), _stream(stream)), "moe_selftest_grid_wait")


def moe_read_device_status(ws, stream=None) -> int:
    return lib().moe_read_device_status(_p(ws), _stream(stream))


def moe_clear_device_status(ws, stream=None):
    _check(lib().moe_clear_device_status(_p(ws), _stream(stream)), "moe_clear_device_status")


# ------------------------------------------------------------- convenience holder
class MoeBlock:
    """A block's config, device-resident weights and workspace for up to max_tokens."""

    def __init__(self, spec, weights: Dict[str, torch.Tensor], max_tokens: int,
                 device: str = "cuda"):
        self.spec = spec
        self.cfg = config_from_spec(spec)
        _check(moe_config_validate(self.cfg), "moe_config_validate")
        self.weights = {k: v.to(device, non_blocking=False).contiguous() for k, v in weights.items()}
        self.w = weights_struct(self.weights)
        _check(moe_weights_validate(self.cfg, self.w), "moe_weights_validate")
        self.max_tokens = int(max_tokens)
        self.ws = torch.zeros(moe_workspace_size(self.cfg, self.max_tokens), dtype=torch.uint8,
                              device=device)
        self.act_dtype = torch.float32 if spec.act_dtype == "f32" else torch.bfloat16

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.spec.hidden), dtype=self.act_dtype, device=x.device)
        moe_block_forward(self.cfg, self.w, x, T, y, self.ws, stream)
        return y

    def device_status(self) -> int:
        return moe_read_device_status(self.ws)
