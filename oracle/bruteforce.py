"""Dense-masked brute-force evaluator of the MoE block -- TEST INFRASTRUCTURE.

A second formulation, written independently of moe_oracle.c, for tiny inputs:
every expert runs on every token, and the routed output is
    y_r[t] = sum_e mask[t, e] * weight[t, e] * FFN_e(u[t])
with mask[t, e] = 1 iff e is among token t's top-k selection keys. The block
structure follows the same pages (Klear PR items 2-3; ferrox latent_moe.rs
module doc; libmir-metal clamped_routed forward), but every step here is a
whole-array numpy operation over all experts at once, so a slip in the
per-token loops of the C oracle does not repeat here.
"""
from __future__ import annotations

from typing import Dict

import numpy as np


def _decode(a: np.ndarray) -> np.ndarray:
    """Stored tensor -> float64 (bf16 bit patterns are widened to f32 first)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _dequant(q: np.ndarray, s: np.ndarray, z: np.ndarray, group: int) -> np.ndarray:
    """Packed 4-bit affine planes [..., K/8] -> float64 [..., K]."""
    shifts = np.arange(8, dtype=np.uint32) * 4
    codes = (q[..., None] >> shifts) & 0xF                 # [..., K/8, 8]
    codes = codes.reshape(*q.shape[:-1], q.shape[-1] * 8).astype(np.float64)
    scale = np.repeat(_decode(s), group, axis=-1)
    bias = np.repeat(_decode(z), group, axis=-1)
    return codes * scale + bias


# OCP Microscaling Formats v1.0, FP4 E2M1: the sixteen code values (table of the spec).
_E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                        -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def _dequant_mxfp4(q: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    """Packed MXFP4 planes [..., K/8] with E8M0 scale bytes [..., K/32] -> float64 [..., K]."""
    shifts = np.arange(8, dtype=np.uint32) * 4
    codes = (q[..., None] >> shifts) & 0xF
    codes = codes.reshape(*q.shape[:-1], q.shape[-1] * 8)
    scale = np.repeat(np.exp2(sbytes.astype(np.float64) - 127.0), 32, axis=-1)
    return _E2M1_TABLE[codes] * scale


def _dense(spec, w, name):
    """A non-routed plane (router, shared, latent): activation dtype, or 4-bit affine words
    with their own scales / biases when the spec quantises the dense parts."""
    if spec.dense_format == "q4":
        stem = name[:-2]
        return _dequant(w[name], w[stem + "_s"], w[stem + "_z"], spec.dense_group_size)
    return _decode(w[name])


def _plane(spec, w, name):
    if spec.weight_format == "mxfp4":
        return _dequant_mxfp4(w[name], w[name[:-2] + "_s"])
    if spec.weight_format == "q4":
        stem = name[:-2]
        return _dequant(w[name], w[stem + "_s"], w[stem + "_z"], spec.group_size)
    return _decode(w[name])


def _sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def _act(spec, g, v):
    if spec.activation == "swiglu":
        return g * _sigmoid(g) * v
    lim = spec.swiglu_limit
    gc = np.minimum(g, lim)
    vc = np.clip(v, -lim, lim)
    return gc * _sigmoid(spec.swiglu_alpha * gc) * (vc + 1.0)


def _topk_mask(keys: np.ndarray, k: int) -> np.ndarray:
    """mask[t, e] for the k largest keys; equal keys rank the lower index first."""
    T, E = keys.shape
    # lexsort: last key is primary -> sort by -key, then by expert index.
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -keys), axis=-1)
    mask = np.zeros((T, E), dtype=bool)
    np.put_along_axis(mask, order[:, :k], True, axis=-1)
    return mask


def forward(spec, weights: Dict[str, np.ndarray], x: np.ndarray) -> Dict[str, np.ndarray]:
    """Dense evaluation of every token; returns y [T, H], mask [T, E], weight [T, E]."""
    X = _decode(x)
    T, H = X.shape
    E, k, I = spec.num_experts, spec.top_k, spec.intermediate
    logits = X @ _dense(spec, weights, "router_w").T
    if spec.has_router_bias:
        logits = logits + _decode(weights["router_b"])
    if spec.scoring == "softmax_all":
        ex = np.exp(logits - logits.max(axis=1, keepdims=True))
        score = ex / ex.sum(axis=1, keepdims=True)
    elif spec.scoring == "sigmoid":
        score = _sigmoid(logits)
    else:
        score = logits
    keys = score + (_decode(weights["selection_bias"]) if spec.has_selection_bias else 0.0)
    mask = _topk_mask(keys, k)
    if spec.scoring == "softmax_topk":
        masked = np.where(mask, logits, -np.inf)
        ex = np.exp(masked - masked.max(axis=1, keepdims=True))
        weight = ex / ex.sum(axis=1, keepdims=True)
    else:
        weight = np.where(mask, score, 0.0)
    if spec.norm_topk_prob:
        weight = weight / weight.sum(axis=1, keepdims=True)
    weight = weight * spec.routed_scaling_factor

    U = X @ _dense(spec, weights, "latent_down_w").T if spec.latent_dim else X   # [T, K]
    if spec.gate_up_interleaved:
        gu = _plane(spec, weights, "gate_up_w")                              # [E, 2I, K]
        Wg, Wu = gu[:, 0::2, :], gu[:, 1::2, :]
    else:
        Wg, Wu = _plane(spec, weights, "gate_w"), _plane(spec, weights, "up_w")
    Wd = _plane(spec, weights, "down_w")                                     # [E, K, I]
    G = np.einsum("tk,eik->eti", U, Wg)
    V = np.einsum("tk,eik->eti", U, Wu)
    if spec.has_expert_bias:
        if spec.gate_up_interleaved:
            b = _decode(weights["gate_up_b"])
            G, V = G + b[:, None, 0::2], V + b[:, None, 1::2]
        else:
            G = G + _decode(weights["gate_b"])[:, None, :]
            V = V + _decode(weights["up_b"])[:, None, :]
    O = np.einsum("eti,eki->etk", _act(spec, G, V), Wd)                      # [E, T, K]
    if spec.has_expert_bias:
        O = O + _decode(weights["down_b"])[:, None, :]
    Yr = np.einsum("te,etk->tk", weight, O)
    if spec.latent_dim:
        if spec.latent_use_norm:
            rms = np.sqrt(np.mean(Yr * Yr, axis=1, keepdims=True) + spec.rms_eps)
            Yr = Yr / rms * _decode(weights["latent_norm_w"])
        Yr = Yr @ _dense(spec, weights, "latent_up_w").T
    coef = np.zeros((T, 2))
    if spec.shared_mode == "none":
        Y = Yr
    else:
        S = _act(spec, X @ _dense(spec, weights, "shared_gate_w").T,
                 X @ _dense(spec, weights, "shared_up_w").T) @ _dense(spec, weights, "shared_down_w").T
        if spec.shared_mode == "add":
            Y = Yr + S
        else:
            c = X @ _decode(weights["coef_w"]).T + _decode(weights["coef_b"])
            ex = np.exp(c - c.max(axis=1, keepdims=True))
            coef = ex / ex.sum(axis=1, keepdims=True)
            Y = Yr * coef[:, :1] + S * coef[:, 1:]
    return {"y": Y, "mask": mask, "weight": weight, "keys": keys, "coef": coef}
