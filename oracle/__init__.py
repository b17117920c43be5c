"""fp64 CPU oracle of the sparse MoE FFN block forward -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package. It shares no code with the CUDA library and never calls it.

Two independent formulations live here:
  * moe_oracle.c -- the plain per-token definition in double precision
    (loaded through ctypes from an in-tree build, OpenMP over tokens);
  * bruteforce.py -- a numpy dense-masked evaluator for tiny inputs.

Each function cites the page passage it follows (see moe_oracle.c's header).
The pins that tie these to the pages and to mathematics are in
tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")

_SCORING = {"softmax_all": 0, "sigmoid": 1, "softmax_topk": 2}
_ACT = {"swiglu": 0, "swiglu_clamped": 1}
_DT = {"f32": 0, "bf16": 1, "q4": 2, "mxfp4": 3}
_SHARED = {"none": 0, "add": 1, "blend": 2}


class OrcConfig(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("num_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("intermediate", ctypes.c_int32),
        ("scoring", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_double),
        ("activation", ctypes.c_int32),
        ("swiglu_limit", ctypes.c_double), ("swiglu_alpha", ctypes.c_double),
        ("gate_up_interleaved", ctypes.c_int32), ("has_expert_bias", ctypes.c_int32),
        ("has_router_bias", ctypes.c_int32), ("has_selection_bias", ctypes.c_int32),
        ("act_dtype", ctypes.c_int32), ("weight_format", ctypes.c_int32),
        ("group_size", ctypes.c_int32),
        ("shared_mode", ctypes.c_int32), ("shared_intermediate", ctypes.c_int32),
        ("latent_dim", ctypes.c_int32), ("latent_use_norm", ctypes.c_int32),
        ("rms_eps", ctypes.c_double),
        ("dense_weight_format", ctypes.c_int32), ("dense_group_size", ctypes.c_int32),
    ]


_WEIGHT_FIELDS = [
    "router_w", "router_b", "selection_bias", "coef_w", "coef_b",
    "gate_w", "up_w", "gate_up_w", "gate_b", "up_b", "gate_up_b", "down_w", "down_b",
    "gate_s", "gate_z", "up_s", "up_z", "down_s", "down_z",
    "shared_gate_w", "shared_up_w", "shared_down_w",
    "latent_down_w", "latent_up_w", "latent_norm_w",
    "gate_up_s", "gate_up_z",
    "router_s", "router_z", "shared_gate_s", "shared_gate_z", "shared_up_s", "shared_up_z",
    "shared_down_s", "shared_down_z", "latent_down_s", "latent_down_z", "latent_up_s", "latent_up_z",
]


class OrcWeights(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _WEIGHT_FIELDS]


def build(force: bool = False) -> str:
    """Compile the oracle in-tree with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64p = ctypes.POINTER(ctypes.c_int64)
        i32p = ctypes.POINTER(ctypes.c_int32)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.orc_forward.argtypes = [ctypes.POINTER(OrcConfig), ctypes.POINTER(OrcWeights),
                                    ctypes.c_void_p, ctypes.c_int64, i64p, ctypes.c_int64,
                                    dp, i32p, dp, dp, dp, dp, ctypes.c_int32]
        lib.orc_forward.restype = ctypes.c_int
        lib.orc_forward_with_indices.argtypes = [ctypes.POINTER(OrcConfig),
                                                 ctypes.POINTER(OrcWeights), ctypes.c_void_p,
                                                 ctypes.c_int64, ctypes.c_int64, i32p, dp, dp]
        lib.orc_forward_with_indices.restype = ctypes.c_int
        lib.orc_permute.argtypes = [i32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                    i32p, i32p, i32p]
        lib.orc_permute.restype = None
        lib.orc_activation.argtypes = [ctypes.c_int32, ctypes.c_double, ctypes.c_double,
                                       ctypes.c_double, ctypes.c_double]
        lib.orc_activation.restype = ctypes.c_double
        lib.orc_dequant_q4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int64, ctypes.c_int32, ctypes.c_int64,
                                       ctypes.c_int64]
        lib.orc_dequant_q4.restype = ctypes.c_double
        lib.orc_dequant_mxfp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int64]
        lib.orc_dequant_mxfp4.restype = ctypes.c_double
        lib.orc_max_threads.argtypes = []
        lib.orc_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().orc_max_threads())


def _config(spec) -> OrcConfig:
    return OrcConfig(
        hidden=spec.hidden, num_experts=spec.num_experts, top_k=spec.top_k,
        intermediate=spec.intermediate, scoring=_SCORING[spec.scoring],
        norm_topk_prob=int(spec.norm_topk_prob),
        routed_scaling_factor=float(spec.routed_scaling_factor),
        activation=_ACT[spec.activation], swiglu_limit=float(spec.swiglu_limit),
        swiglu_alpha=float(spec.swiglu_alpha),
        gate_up_interleaved=int(spec.gate_up_interleaved),
        has_expert_bias=int(spec.has_expert_bias), has_router_bias=int(spec.has_router_bias),
        has_selection_bias=int(spec.has_selection_bias), act_dtype=_DT[spec.act_dtype],
        weight_format=_DT[spec.weight_format], group_size=spec.group_size,
        shared_mode=_SHARED[spec.shared_mode], shared_intermediate=spec.shared_intermediate,
        latent_dim=spec.latent_dim, latent_use_norm=int(spec.latent_use_norm),
        rms_eps=float(spec.rms_eps),
        dense_weight_format=_DT["q4"] if spec.dense_format == "q4" else _DT[spec.act_dtype],
        dense_group_size=spec.dense_group_size)


def _check_storage(a: np.ndarray) -> np.ndarray:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    assert a.dtype in (np.float32, np.uint16, np.uint32, np.uint8), a.dtype
    return a


def _weights(w: Dict[str, np.ndarray]) -> OrcWeights:
    ow = OrcWeights()
    for f in _WEIGHT_FIELDS:
        a = w.get(f)
        if a is not None:
            setattr(ow, f, _check_storage(a).ctypes.data)
    return ow


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def forward(spec, weights: Dict[str, np.ndarray], x: np.ndarray,
            tokens: Optional[Sequence[int]] = None, route_only: bool = False,
            threads: int = 0) -> Dict[str, np.ndarray]:
    """Evaluate the block on the listed tokens of x [T, hidden].

    `weights` and `x` are bit-exact numpy views of the stored tensors
    (float32, bf16 as uint16, packed 4-bit words as uint32). Returns y
    [n, hidden] (absent when route_only), idx [n, k] (descending selection
    key), w [n, k] combine weights, coef [n, 2] (blend only, else zeros),
    keys [n, E] selection keys and logits [n, E].
    """
    lib = _load()
    x = _check_storage(x)
    T = x.shape[0]
    toks = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, dtype=np.int64)
    toks = np.ascontiguousarray(toks)
    n, H, E, k = len(toks), spec.hidden, spec.num_experts, spec.top_k
    y = None if route_only else np.zeros((n, H), dtype=np.float64)
    idx = np.zeros((n, k), dtype=np.int32)
    wts = np.zeros((n, k), dtype=np.float64)
    coef = np.zeros((n, 2), dtype=np.float64)
    keys = np.zeros((n, E), dtype=np.float64)
    logits = np.zeros((n, E), dtype=np.float64)
    cfg = _config(spec)
    ow = _weights(weights)
    rc = lib.orc_forward(ctypes.byref(cfg), ctypes.byref(ow), x.ctypes.data, T,
                         _ptr(toks, ctypes.c_int64), n,
                         None if y is None else _ptr(y, ctypes.c_double),
                         _ptr(idx, ctypes.c_int32), _ptr(wts, ctypes.c_double),
                         _ptr(coef, ctypes.c_double), _ptr(keys, ctypes.c_double),
                         _ptr(logits, ctypes.c_double), int(threads))
    if rc != 0:
        raise ValueError("oracle: token index out of range")
    out = {"idx": idx, "w": wts, "coef": coef, "keys": keys, "logits": logits}
    if y is not None:
        out["y"] = y
    return out


def forward_with_indices(spec, weights, x: np.ndarray, t: int, idx: Sequence[int]):
    """Token t of x evaluated with the given expert set; returns (y [H], w [k])."""
    lib = _load()
    forced = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    assert forced.shape == (spec.top_k,)
    y = np.zeros(spec.hidden, dtype=np.float64)
    wts = np.zeros(spec.top_k, dtype=np.float64)
    cfg = _config(spec)
    ow = _weights(weights)
    rc = lib.orc_forward_with_indices(ctypes.byref(cfg), ctypes.byref(ow),
                                      _check_storage(x).ctypes.data, x.shape[0], int(t),
                                      _ptr(forced, ctypes.c_int32), _ptr(y, ctypes.c_double),
                                      _ptr(wts, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle: bad token or expert index")
    return y, wts


def permute(idx: np.ndarray, num_experts: int):
    """Stable counting sort of slots t*k+j by expert: (offsets, sorted_slot, slot_pos)."""
    lib = _load()
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    T, k = idx.shape
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    sorted_slot = np.zeros(T * k, dtype=np.int32)
    slot_pos = np.zeros(T * k, dtype=np.int32)
    lib.orc_permute(_ptr(idx, ctypes.c_int32), T, k, num_experts,
                    _ptr(offsets, ctypes.c_int32), _ptr(sorted_slot, ctypes.c_int32),
                    _ptr(slot_pos, ctypes.c_int32))
    return offsets, sorted_slot, slot_pos


def activation(kind: str, g: float, v: float, limit: float = 7.0, alpha: float = 1.702) -> float:
    return float(_load().orc_activation(_ACT[kind], g, v, limit, alpha))


def dequant_q4(q: np.ndarray, scales: np.ndarray, biases: np.ndarray, cols: int,
               group_size: int, row: int, col: int) -> float:
    q = _check_storage(q)
    return float(_load().orc_dequant_q4(q.ctypes.data, _check_storage(scales).ctypes.data,
                                        _check_storage(biases).ctypes.data, cols, group_size,
                                        row, col))


def dequant_mxfp4(q: np.ndarray, scales: np.ndarray, cols: int, row: int, col: int) -> float:
    """One MXFP4 weight W[row, col] (E2M1 element times its block's E8M0 scale)."""
    q = _check_storage(q)
    return float(_load().orc_dequant_mxfp4(q.ctypes.data, _check_storage(scales).ctypes.data, cols, row, col))
