"""Seeded sweep of random tiny block variants: the sparse per-token oracle equals the
dense-masked brute-force evaluator on every combination of options.

The fixed variants elsewhere each exercise one branch of the block; this sweep draws the
options together (scoring, selection and router biases, renormalisation, activation,
interleaved planes, expert biases, weight format, 4-bit dense planes, shared add / blend,
latent with or without the norm) so that an interaction between two branches that no fixed variant
combines still meets an independent evaluation. Shapes stay tiny: the brute force runs
every expert on every token.
"""
import numpy as np
import pytest

import oracle
from oracle import bruteforce
from sparse_moe_ffn_gemv_b200 import inputs
from sparse_moe_ffn_gemv_b200.inputs import MoeSpec

N_SPECS = 32


def _random_spec(i: int) -> MoeSpec:
    rng = np.random.default_rng(7000 + i)
    fmt = str(rng.choice(["f32", "bf16", "q4", "mxfp4"]))
    four_bit = fmt in ("q4", "mxfp4")
    dense_q4 = fmt != "f32" and bool(rng.random() < 0.35)   # 4-bit router / shared / latent
    E = int(rng.integers(1, 10))
    k = int(rng.integers(1, E + 1))
    latent = bool(rng.random() < 0.3)
    widths = [32, 64] if four_bit else [8, 16, 24, 32]
    hidden = int(rng.choice([8, 16, 24, 40, 48]))
    if dense_q4 or (four_bit and not latent):
        hidden = int(rng.choice([32, 64]))                  # a 4-bit plane's input width
    L = int(rng.choice([32, 64] if (four_bit or dense_q4) else widths)) if latent else 0
    I = int(rng.choice(widths))
    shared = str(rng.choice(["none", "add", "blend"]))
    Is = (32 if dense_q4 else int(rng.choice([8, 16]))) if shared != "none" else 0
    return MoeSpec(
        name=f"sweep{i}", config_id=7000 + i, hidden=hidden, num_experts=E, top_k=k, intermediate=I,
        scoring=str(rng.choice(["softmax_all", "sigmoid", "softmax_topk"])),
        norm_topk_prob=bool(rng.random() < 0.5),
        activation=str(rng.choice(["swiglu", "swiglu_clamped"])),
        gate_up_interleaved=bool(rng.random() < 0.5),
        has_expert_bias=bool(rng.random() < 0.5),
        has_router_bias=bool(rng.random() < 0.3),
        has_selection_bias=bool(rng.random() < 0.5),
        act_dtype="f32" if fmt == "f32" else "bf16", weight_format=fmt,
        group_size=32 if fmt == "mxfp4" else int(rng.choice([32] if min(I, L or hidden) < 64 else [32, 64])),
        shared_mode=shared, shared_intermediate=Is,
        latent_dim=L, latent_use_norm=bool(latent and rng.random() < 0.7), rms_eps=1e-6,
        dense_format="q4" if dense_q4 else "act", dense_group_size=32)


SPECS = [_random_spec(i) for i in range(N_SPECS)]


def _label(s: MoeSpec) -> str:
    return (f"{s.name}-{s.weight_format}-E{s.num_experts}k{s.top_k}-{s.scoring}-{s.activation}"
            f"{'-il' if s.gate_up_interleaved else ''}{'-lat' if s.latent_dim else ''}-{s.shared_mode}"
            f"{'-dq4' if s.dense_format == 'q4' else ''}")


@pytest.mark.parametrize("spec", SPECS, ids=_label)
def test_random_variant_oracle_equals_bruteforce(spec):
    rng = np.random.default_rng(spec.config_id)
    T = int(rng.integers(1, 10))
    scale = 30.0 if spec.activation == "swiglu_clamped" else 1.0
    w = {k: inputs.to_numpy_storage(v) for k, v in inputs.make_weights(spec, threads=2).items()}
    x = inputs.to_numpy_storage(inputs.make_x(spec, T, scale))
    o = oracle.forward(spec, w, x)
    b = bruteforce.forward(spec, w, x)
    mag = np.abs(b["y"]).max()
    assert np.all(np.isfinite(o["y"]))
    np.testing.assert_allclose(o["y"], b["y"], rtol=1e-10, atol=1e-12 * max(mag, 1e-300))
    for t in range(T):
        assert set(o["idx"][t]) == set(np.nonzero(b["mask"][t])[0])
        np.testing.assert_allclose(o["w"][t], b["weight"][t, o["idx"][t]], rtol=1e-12)
    if spec.shared_mode == "blend":
        np.testing.assert_allclose(o["coef"], b["coef"], rtol=1e-12)


def test_sweep_covers_every_option():
    seen = {f: {getattr(s, f) for s in SPECS} for f in
            ("weight_format", "scoring", "activation", "gate_up_interleaved", "has_expert_bias",
             "has_router_bias", "has_selection_bias", "norm_topk_prob", "shared_mode", "latent_use_norm",
             "dense_format")}
    assert seen["weight_format"] == {"f32", "bf16", "q4", "mxfp4"}
    assert seen["scoring"] == {"softmax_all", "sigmoid", "softmax_topk"}
    assert seen["shared_mode"] == {"none", "add", "blend"}
    for f in ("activation", "gate_up_interleaved", "has_expert_bias", "has_router_bias",
              "has_selection_bias", "norm_topk_prob", "latent_use_norm", "dense_format"):
        assert len(seen[f]) == 2, f
    assert any(s.latent_dim for s in SPECS) and any(s.weight_format in ("q4", "mxfp4") and s.gate_up_interleaved
                                                     for s in SPECS)
