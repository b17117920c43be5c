"""Block configurations and seeded synthetic inputs for the sparse MoE FFN block.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests. It holds shapes, seeds and the synthetic checkpoint encoder (the 4-bit
affine quantiser that stands in for a converted checkpoint); it holds none of
the block's forward arithmetic.

Shapes follow the pages' models:
  * the Klear-46B-A2.5B sparse block (hidden 2048, 256 experts, top-8, one
    shared expert) -- "Klear sparse MoE family" PR, opening paragraph;
  * Kimi K3's latent MoE (hidden 7168, latent 3584) -- ferrox latent_moe.rs,
    module doc comment;
  * a clamped-SwiGLU routed family with a fused interleaved gate_up plane and
    linear biases -- libmir-metal clamped_routed/experts/mod.rs, ExpertLayout;
  * 4-bit affine stacked expert planes with group 64 -- mlxcel issue #974,
    "What exists" / the Jamba2-Mini checkpoint description.

Recipe (every tensor is drawn independently so that generation can run in
parallel and weights do not depend on the token count):
  generator seed = 20261202 + 1000*config_id + crc32(tensor name) (+ T for x)
  x ~ N(0,1); all weights ~ N(0, 0.02); the select-only expert bias ~ N(0, 0.1);
  linear biases ~ N(0, 0.02); the RMSNorm weight = 1 + N(0, 0.1).
  Draws are fp32, then cast to the storage dtype.
"""
from __future__ import annotations

import dataclasses
import zlib
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np
import torch

# Enum codes; the same integers appear in include/moe.h.
SCORING = {"softmax_all": 0, "sigmoid": 1, "softmax_topk": 2}
ACTIVATION = {"swiglu": 0, "swiglu_clamped": 1}
DTYPE = {"f32": 0, "bf16": 1, "q4": 2, "mxfp4": 3}
SHARED = {"none": 0, "add": 1, "blend": 2}


@dataclasses.dataclass(frozen=True)
class MoeSpec:
    name: str
    config_id: int
    hidden: int
    num_experts: int
    top_k: int
    intermediate: int
    scoring: str = "sigmoid"
    norm_topk_prob: bool = False
    routed_scaling_factor: float = 1.0
    activation: str = "swiglu"
    swiglu_limit: float = 7.0
    swiglu_alpha: float = 1.702
    gate_up_interleaved: bool = False
    has_expert_bias: bool = False
    has_router_bias: bool = False
    has_selection_bias: bool = False
    act_dtype: str = "bf16"
    weight_format: str = "bf16"
    group_size: int = 64
    bits: int = 4
    shared_mode: str = "none"
    shared_intermediate: int = 0
    latent_dim: int = 0
    latent_use_norm: bool = False
    rms_eps: float = 1e-6
    # non-routed planes (router, shared expert, latent projections): "act" = the activation
    # dtype, "q4" = 4-bit affine with dense_group_size (the 2-row blend head stays in act)
    dense_format: str = "act"
    dense_group_size: int = 64
    token_counts: tuple = ()

    @property
    def expert_in(self) -> int:
        """K of the routed experts: the latent width when latent, else hidden."""
        return self.latent_dim if self.latent_dim else self.hidden

    def replace(self, **kw) -> "MoeSpec":
        return dataclasses.replace(self, **kw)


# The five workloads.
TINY_F32 = MoeSpec(
    name="tiny_f32", config_id=1, hidden=64, num_experts=8, top_k=2, intermediate=32,
    scoring="softmax_all", norm_topk_prob=False, act_dtype="f32", weight_format="f32",
    token_counts=(16,))
KLEAR_BF16 = MoeSpec(
    name="klear_bf16", config_id=2, hidden=2048, num_experts=256, top_k=8, intermediate=768,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True,
    shared_mode="blend", shared_intermediate=768, token_counts=(1, 8, 64, 4096))
KLEAR_Q4 = KLEAR_BF16.replace(name="klear_q4", config_id=3, weight_format="q4",
                              token_counts=(1, 32, 2048))
CLAMPED_BF16 = MoeSpec(
    name="clamped_bf16", config_id=4, hidden=2880, num_experts=128, top_k=4, intermediate=2880,
    scoring="softmax_topk", activation="swiglu_clamped", gate_up_interleaved=True,
    has_expert_bias=True, token_counts=(1, 8192))
LATENT_BF16 = MoeSpec(
    name="latent_bf16", config_id=5, hidden=7168, num_experts=384, top_k=8, intermediate=2048,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True,
    shared_mode="add", shared_intermediate=2048, latent_dim=3584, latent_use_norm=True,
    rms_eps=1e-6, token_counts=(1, 128, 8192))

# The clamped-routed family with MXFP4 expert planes in the split/u32 layout (libmir-metal
# clamped_routed: gate, up and down blocks with scales and biases; not interleaved).
CLAMPED_MXFP4 = CLAMPED_BF16.replace(name="clamped_mxfp4", config_id=6, weight_format="mxfp4",
                                     gate_up_interleaved=False, group_size=32, token_counts=(1, 8, 8192))
# The same family in the native MXFP4 layout (libmir-metal clamped_routed ExpertLayout::Native):
# one interleaved gate_up block plane (row 2i gate, 2i + 1 up) with its scales and bias.
CLAMPED_MXFP4_NATIVE = CLAMPED_MXFP4.replace(name="clamped_mxfp4_native", config_id=7,
                                             gate_up_interleaved=True)

# The 4-bit Klear block with its dense planes 4-bit as well (router, shared expert; the 2-row
# blend head stays bf16), as a 4-bit checkpoint quantises its dense projections too (mlxcel
# issue #974, the Jamba study).
KLEAR_Q4_DENSE = KLEAR_Q4.replace(name="klear_q4_dense", config_id=8, dense_format="q4", dense_group_size=64,
                                  token_counts=(1, 32, 2048))

WORKLOADS = {s.name: s for s in (TINY_F32, KLEAR_BF16, KLEAR_Q4, CLAMPED_BF16, LATENT_BF16, CLAMPED_MXFP4,
                                 CLAMPED_MXFP4_NATIVE, KLEAR_Q4_DENSE)}

BASE_SEED = 20261202


def _seed(spec: MoeSpec, name: str, extra: int = 0) -> int:
    return (BASE_SEED + 1000 * spec.config_id + zlib.crc32(name.encode()) + extra) % (2 ** 63)


def _normal(shape, std: float, seed: int, mean: float = 0.0) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def _storage(t: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return t.contiguous()
    return t.to(torch.bfloat16).contiguous()


def quantize_affine_q4(w: torch.Tensor, group_size: int):
    """Encode fp32 planes [..., K] as a synthetic 4-bit affine checkpoint.

    Per group of `group_size` consecutive input elements: scale = (max-min)/15
    and bias = min, both rounded to bf16 first; q = clamp(round((w-bias)/scale),
    0, 15). Eight codes pack into one uint32, element j of a row at bits
    4*(j mod 8) of word j/8. Returns (packed words [..., K/8] as int32 bit patterns, scales bf16
    [..., K/group], biases bf16 [..., K/group]).
    """
    *lead, k = w.shape
    assert k % group_size == 0 and k % 8 == 0
    g = w.reshape(*lead, k // group_size, group_size)
    mn = g.amin(dim=-1)
    mx = g.amax(dim=-1)
    scale = ((mx - mn) / 15.0).clamp_min(1e-8).to(torch.bfloat16)
    bias = mn.to(torch.bfloat16)
    q = torch.round((g - bias.float().unsqueeze(-1)) / scale.float().unsqueeze(-1)).clamp_(0, 15)
    q = q.to(torch.int64).reshape(*lead, k // 8, 8)
    shifts = torch.arange(8, dtype=torch.int64) * 4
    packed = (q << shifts).sum(dim=-1)
    packed = packed.bitwise_and(0xFFFFFFFF).numpy().astype(np.uint32).view(np.int32)
    # torch has no general uint32 arithmetic: the words travel as int32 bit patterns.
    return torch.from_numpy(packed.copy()), scale.contiguous(), bias.contiguous()


# E2M1 magnitudes by the low three bits of a code (OCP Microscaling Formats v1.0), and the
# midpoints between neighbours (a magnitude rounds to the index of the first midpoint >= it).
_E2M1 = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E2M1_MID = (_E2M1[1:] + _E2M1[:-1]) / 2


def quantize_mxfp4(w: torch.Tensor):
    """Encode fp32 planes [..., K] as a synthetic MXFP4 checkpoint (OCP MX v1.0).

    Per block of 32 consecutive input elements: the shared E8M0 scale is 2^x with
    x = floor(log2(max |w|)) - 2 (the largest E2M1 exponent), stored as the byte x + 127;
    each element is w / 2^x rounded to the nearest E2M1 value (ties to the smaller
    magnitude), clamped to +-6; code = sign bit 8 | magnitude index. Codes pack as the
    4-bit planes do: element j of a row at bits 4*(j mod 8) of word j/8. Returns (packed
    words [..., K/8] as int32 bit patterns, scale bytes uint8 [..., K/32]).
    """
    *lead, k = w.shape
    assert k % 32 == 0
    g = w.reshape(*lead, k // 32, 32)
    amax = g.abs().amax(dim=-1).clamp_min(2.0 ** -120)
    x = torch.floor(torch.log2(amax)) - 2.0
    sbyte = (x + 127).clamp(1, 254)
    v = (g / torch.exp2(sbyte - 127).unsqueeze(-1)).clamp(-6.0, 6.0)
    idx = torch.bucketize(v.abs(), _E2M1_MID)  # nearest E2M1 magnitude; a tie keeps the smaller
    code = idx + torch.where(v < 0, 8, 0) * (idx > 0)
    code = code.to(torch.int64).reshape(*lead, k // 8, 8)
    shifts = torch.arange(8, dtype=torch.int64) * 4
    packed = (code << shifts).sum(dim=-1)
    packed = packed.bitwise_and(0xFFFFFFFF).numpy().astype(np.uint32).view(np.int32)
    return torch.from_numpy(packed.copy()), sbyte.to(torch.uint8).contiguous()


def _expert_plane(spec: MoeSpec, name: str, rows: int, cols: int, pool) -> Dict[str, torch.Tensor]:
    """One stacked expert projection [E, rows, cols] in the spec's weight format.

    Each expert is drawn from its own generator so the draws run in parallel.
    """
    e_count = spec.num_experts

    def one(e):
        w = _normal((rows, cols), 0.02, _seed(spec, f"{name}/{e}"))
        if spec.weight_format == "q4":
            return quantize_affine_q4(w, spec.group_size)
        if spec.weight_format == "mxfp4":
            return quantize_mxfp4(w)
        return (_storage(w, spec.weight_format),)

    parts = list(pool.map(one, range(e_count)))
    if spec.weight_format == "mxfp4":  # "gate_w" -> "gate_s" (E8M0 scale bytes)
        return {name: torch.stack([p[0] for p in parts]), name[:-2] + "_s": torch.stack([p[1] for p in parts])}
    if spec.weight_format == "q4":
        stem = name[:-2]  # "gate_w" -> companions "gate_s" (scales), "gate_z" (biases)
        return {name: torch.stack([p[0] for p in parts]),
                stem + "_s": torch.stack([p[1] for p in parts]),
                stem + "_z": torch.stack([p[2] for p in parts])}
    return {name: torch.stack([p[0] for p in parts])}


def _dense_plane(spec: MoeSpec, name: str, rows: int, cols: int) -> Dict[str, torch.Tensor]:
    """One non-routed plane [rows, cols] ~ N(0, 0.02): in the activation dtype, or (dense
    format q4) the same draw encoded 4-bit affine, "router_w" -> companions "router_s",
    "router_z"."""
    w = _normal((rows, cols), 0.02, _seed(spec, name))
    if spec.dense_format == "q4":
        q, sc, bi = quantize_affine_q4(w, spec.dense_group_size)
        return {name: q, name[:-2] + "_s": sc, name[:-2] + "_z": bi}
    return {name: _storage(w, spec.act_dtype)}


def make_weights(spec: MoeSpec, threads: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All block weights on the CPU, keyed by the C ABI's moe_weights field names."""
    H, E, I = spec.hidden, spec.num_experts, spec.intermediate
    K = spec.expert_in
    act = spec.act_dtype
    w: Dict[str, torch.Tensor] = {}
    w.update(_dense_plane(spec, "router_w", E, H))
    if spec.has_router_bias:
        w["router_b"] = _storage(_normal((E,), 0.02, _seed(spec, "router_b")), act)
    if spec.has_selection_bias:
        w["selection_bias"] = _normal((E,), 0.1, _seed(spec, "selection_bias"))
    if spec.shared_mode == "blend":
        w["coef_w"] = _storage(_normal((2, H), 0.02, _seed(spec, "coef_w")), act)
        w["coef_b"] = _storage(_normal((2,), 0.02, _seed(spec, "coef_b")), act)
    with ThreadPoolExecutor(max_workers=threads or max(1, torch.get_num_threads())) as pool:
        if spec.gate_up_interleaved:
            w.update(_expert_plane(spec, "gate_up_w", 2 * I, K, pool))
        else:
            w.update(_expert_plane(spec, "gate_w", I, K, pool))
            w.update(_expert_plane(spec, "up_w", I, K, pool))
        w.update(_expert_plane(spec, "down_w", K, I, pool))
    if spec.has_expert_bias:
        if spec.gate_up_interleaved:
            w["gate_up_b"] = _storage(_normal((E, 2 * I), 0.02, _seed(spec, "gate_up_b")), act)
        else:
            w["gate_b"] = _storage(_normal((E, I), 0.02, _seed(spec, "gate_b")), act)
            w["up_b"] = _storage(_normal((E, I), 0.02, _seed(spec, "up_b")), act)
        w["down_b"] = _storage(_normal((E, K), 0.02, _seed(spec, "down_b")), act)
    if spec.shared_mode != "none":
        Is = spec.shared_intermediate
        w.update(_dense_plane(spec, "shared_gate_w", Is, H))
        w.update(_dense_plane(spec, "shared_up_w", Is, H))
        w.update(_dense_plane(spec, "shared_down_w", H, Is))
    if spec.latent_dim:
        L = spec.latent_dim
        w.update(_dense_plane(spec, "latent_down_w", L, H))
        w.update(_dense_plane(spec, "latent_up_w", H, L))
        if spec.latent_use_norm:
            w["latent_norm_w"] = _storage(
                _normal((L,), 0.1, _seed(spec, "latent_norm_w"), mean=1.0), act)
    return w


def make_x(spec: MoeSpec, T: int, scale: float = 1.0) -> torch.Tensor:
    """Block input [T, hidden] ~ N(0, scale^2) in the activation dtype."""
    x = _normal((T, spec.hidden), scale, _seed(spec, "x", extra=T))
    return _storage(x, spec.act_dtype)


def to_numpy_storage(t: torch.Tensor) -> np.ndarray:
    """Bit-exact numpy view of a stored tensor: bf16 -> uint16, f32 -> float32,
    packed 4-bit words (int32) -> uint32, MXFP4 scale bytes -> uint8."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    return t.numpy()
