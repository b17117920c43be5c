"""Tiny block variants used by the oracle pins and the small parity cases.

Each variant exercises one branch of the block: sigmoid routing with a
select-only bias and the shared-expert blend (Klear PR items 2-3), softmax
over the top-k logits with clamped SwiGLU on an interleaved gate_up plane with
biases (libmir-metal clamped_routed ExpertLayout::DenseFused), 4-bit affine
planes (mlxcel issue #974), the latent variant (ferrox latent_moe.rs), and MXFP4
planes in the clamped family's split and native (interleaved gate_up) layouts
(libmir-metal clamped_routed; element and scale encodings from the OCP Microscaling
Formats v1.0 specification).
"""
import numpy as np

from sparse_moe_ffn_gemv_b200 import inputs
from sparse_moe_ffn_gemv_b200.inputs import MoeSpec

SIG_BLEND = MoeSpec(
    name="t_sig_blend", config_id=101, hidden=48, num_experts=6, top_k=3, intermediate=16,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True,
    shared_mode="blend", shared_intermediate=24)
CLAMPED = MoeSpec(
    name="t_clamped", config_id=102, hidden=40, num_experts=5, top_k=2, intermediate=24,
    scoring="softmax_topk", activation="swiglu_clamped", gate_up_interleaved=True,
    has_expert_bias=True)
Q4 = MoeSpec(
    name="t_q4", config_id=103, hidden=128, num_experts=4, top_k=2, intermediate=64,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True, weight_format="q4",
    group_size=64, shared_mode="blend", shared_intermediate=32)
LATENT = MoeSpec(
    name="t_latent", config_id=104, hidden=48, num_experts=6, top_k=2, intermediate=16,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True, shared_mode="add",
    shared_intermediate=24, latent_dim=24, latent_use_norm=True)
ROUTER_BIAS = MoeSpec(
    name="t_router_bias", config_id=105, hidden=32, num_experts=7, top_k=3, intermediate=8,
    scoring="softmax_all", has_router_bias=True, norm_topk_prob=True, shared_mode="add",
    shared_intermediate=8, act_dtype="f32", weight_format="f32")
SEPARATE_BIAS = MoeSpec(
    name="t_sep_bias", config_id=106, hidden=64, num_experts=4, top_k=2, intermediate=32,
    scoring="sigmoid", norm_topk_prob=False, has_expert_bias=True, weight_format="q4",
    group_size=32)
LATENT_NONORM = LATENT.replace(name="t_latent_nonorm", config_id=107, latent_use_norm=False)
# MXFP4 planes (OCP MX v1.0 encoding) in the clamped family's split layout, with biases
MXFP4 = MoeSpec(
    name="t_mxfp4", config_id=108, hidden=128, num_experts=5, top_k=2, intermediate=64,
    scoring="softmax_topk", activation="swiglu_clamped", has_expert_bias=True,
    weight_format="mxfp4", group_size=32)
# the same family in the native layout: one interleaved gate_up block plane with its scales
# and bias (libmir-metal clamped_routed ExpertLayout::Native)
MXFP4_NATIVE = MXFP4.replace(name="t_mxfp4_native", config_id=109, gate_up_interleaved=True)
# 4-bit affine on an interleaved gate_up plane (its scales and biases interleaved alike)
Q4_INTERLEAVED = MoeSpec(
    name="t_q4_il", config_id=110, hidden=128, num_experts=4, top_k=2, intermediate=64,
    scoring="softmax_topk", activation="swiglu_clamped", gate_up_interleaved=True,
    has_expert_bias=True, weight_format="q4", group_size=32)

# every dense plane 4-bit as well (router, shared expert, latent projections; the blend head
# stays bf16): a 4-bit checkpoint quantises its dense projections too (mlxcel issue #974)
DENSE_Q4 = MoeSpec(
    name="t_dense_q4", config_id=111, hidden=64, num_experts=6, top_k=2, intermediate=32,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True, weight_format="q4",
    group_size=32, shared_mode="add", shared_intermediate=32, latent_dim=32, latent_use_norm=True,
    dense_format="q4", dense_group_size=32)
DENSE_Q4_BLEND = Q4.replace(name="t_dense_q4_blend", config_id=112, dense_format="q4", dense_group_size=32)

# bf16 shapes on which a few hundred tokens give the tensor-core launches 256-token tiles with
# ragged halves: experts holding 129..256 and more than 256 routed rows, dense tails of 188
# rows (clamped family with biases and the blend head; latent block with the add, wide enough
# that its three bf16 intermediates z, h and the normalised latent stay inside the bar: at
# hidden 128 / latent 128 their roundings alone reach 0.022 rms)
WIDE = MoeSpec(
    name="t_wide", config_id=113, hidden=128, num_experts=4, top_k=2, intermediate=128,
    scoring="softmax_topk", activation="swiglu_clamped", gate_up_interleaved=True,
    has_expert_bias=True, shared_mode="blend", shared_intermediate=64)
# 4-bit routed experts with a bf16 shared expert and an odd number of 64-wide K blocks
# (hidden 192): in a batch with more tensor-core tiles than SMs a CTA runs shared-expert bf16
# tiles and then 4-bit tiles, which move its operand-slot barriers an odd number of phases on
Q4_ODD_K = MoeSpec(
    name="t_q4_odd_k", config_id=115, hidden=192, num_experts=8, top_k=2, intermediate=128,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True, weight_format="q4",
    group_size=64, shared_mode="add", shared_intermediate=128)
LATENT_WIDE = MoeSpec(
    name="t_latent_wide", config_id=114, hidden=512, num_experts=6, top_k=2, intermediate=128,
    scoring="sigmoid", has_selection_bias=True, norm_topk_prob=True, shared_mode="add",
    shared_intermediate=128, latent_dim=256, latent_use_norm=True)

ALL = [inputs.TINY_F32, SIG_BLEND, CLAMPED, Q4, LATENT, ROUTER_BIAS, SEPARATE_BIAS,
       LATENT_NONORM, MXFP4, MXFP4_NATIVE, Q4_INTERLEAVED, DENSE_Q4, DENSE_Q4_BLEND]


def np_weights(spec, scale_weights: float = 1.0):
    """Stored weights as bit-exact numpy arrays (the oracle's input form)."""
    w = inputs.make_weights(spec, threads=4)
    return {k: inputs.to_numpy_storage(v) for k, v in w.items()}


def np_x(spec, T, scale=1.0):
    return inputs.to_numpy_storage(inputs.make_x(spec, T, scale))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 values that are exactly representable in bf16 -> bf16 bit patterns."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "value not exact in bf16"
    return (bits >> 16).astype(np.uint16)
