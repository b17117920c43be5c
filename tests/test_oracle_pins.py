"""Pins of the fp64 oracle to what the pages and mathematics fix (CPU only).

Each test names the passage it checks. None of them retypes the oracle's own
formulas: they compare against the independent brute-force evaluator, library
routines (torch / numpy), closed forms and invariants, or values the pages print.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import bruteforce
from sparse_moe_ffn_gemv_b200 import inputs
from tiny_specs import (ALL, CLAMPED, DENSE_Q4, LATENT, LATENT_NONORM, MXFP4, MXFP4_NATIVE, Q4,
                        Q4_INTERLEAVED, ROUTER_BIAS, SIG_BLEND, np_weights, np_x, to_bf16_bits)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _dec(a):
    """Library decode of stored bits to float64 (independent of both oracles)."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    return a.astype(np.float64)


def _x_scale(spec):
    # The clamp at 7 engages only for large pre-activations (clamped variant).
    return 60.0 if spec.activation == "swiglu_clamped" else 1.0


# --- brute force: the sparse per-token oracle == the dense-masked evaluator ---
@pytest.mark.parametrize("spec", ALL, ids=lambda s: s.name)
def test_sparse_oracle_equals_dense_masked_bruteforce(spec):
    T = 7 if spec.name != "tiny_f32" else 16
    w = np_weights(spec)
    x = np_x(spec, T, _x_scale(spec))
    o = oracle.forward(spec, w, x)
    b = bruteforce.forward(spec, w, x)
    scale = np.abs(b["y"]).max()
    assert scale > 0
    np.testing.assert_allclose(o["y"], b["y"], rtol=1e-10, atol=1e-12 * scale)
    for t in range(T):
        assert set(o["idx"][t]) == set(np.nonzero(b["mask"][t])[0])
        np.testing.assert_allclose(o["w"][t], b["weight"][t, o["idx"][t]], rtol=1e-12)
        # idx is ordered by descending selection key
        assert np.all(np.diff(o["keys"][t, o["idx"][t]]) <= 0)
    if spec.shared_mode == "blend":
        np.testing.assert_allclose(o["coef"], b["coef"], rtol=1e-12)


def test_clamp_engages_in_the_clamped_variant():
    """The clamped case above must actually reach the clamp (else it pins nothing)."""
    w = np_weights(CLAMPED)
    x = np_x(CLAMPED, 7, _x_scale(CLAMPED))
    X = _dec(x)
    gu = _dec(w["gate_up_w"])
    pre = np.einsum("tk,erk->etr", X, gu) + _dec(w["gate_up_b"])[:, None, :]
    assert (pre[:, :, 0::2] > 7).any() and (np.abs(pre[:, :, 1::2]) > 7).any()


# --- Klear PR item 2: the shared expert is blended, not added -----------------
def _zero_routed(w):
    w = dict(w)
    w["down_w"] = np.zeros_like(w["down_w"])
    return w


def _set_coef(w, b0, b1, spec):
    w = dict(w)
    w["coef_w"] = np.zeros_like(w["coef_w"])
    w["coef_b"] = to_bf16_bits(np.array([b0, b1])) if spec.act_dtype == "bf16" else \
        np.array([b0, b1], dtype=np.float32)
    return w


def test_blend_is_not_add_and_index1_weights_shared():
    spec = SIG_BLEND
    T = 5
    x = np_x(spec, T)
    w = _zero_routed(np_weights(spec))            # routed branch == 0 exactly
    shared_only = oracle.forward(spec.replace(shared_mode="add"), w, x)["y"]   # = s
    assert np.abs(shared_only).max() > 1e-4
    # coefficient logits (0, 0): coef = (1/2, 1/2) exactly -> y = s / 2, not s
    y = oracle.forward(spec, _set_coef(w, 0.0, 0.0, spec), x)["y"]
    np.testing.assert_allclose(y, 0.5 * shared_only, rtol=1e-14, atol=0)
    assert np.abs(y - shared_only).max() > 0.25 * np.abs(shared_only).max()
    # logits (b0, 0) with b0 = 1.09375 (bf16-exact, ~ln 3): coef[1] = 1 / (1 + e^{b0})
    b0 = 1.09375
    y = oracle.forward(spec, _set_coef(w, b0, 0.0, spec), x)["y"]
    np.testing.assert_allclose(y, shared_only / (1.0 + math.exp(b0)), rtol=1e-13)
    # index 1 weights the shared branch: a large logit there selects s, index 0 selects 0
    y1 = oracle.forward(spec, _set_coef(w, 0.0, 30.0, spec), x)["y"]
    np.testing.assert_allclose(y1, shared_only, rtol=1e-12)
    y0 = oracle.forward(spec, _set_coef(w, 30.0, 0.0, spec), x)["y"]
    assert np.abs(y0).max() < 1e-12 * np.abs(shared_only).max()


def test_blend_with_equal_coefficients_is_half_of_add():
    """coef = (1/2, 1/2): blend(y_r, s) = (y_r + s) / 2 = add / 2, routed branch live."""
    spec = SIG_BLEND
    x = np_x(spec, 6)
    w = _set_coef(np_weights(spec), 0.0, 0.0, spec)
    y_blend = oracle.forward(spec, w, x)["y"]
    y_add = oracle.forward(spec.replace(shared_mode="add"), w, x)["y"]
    y_none = oracle.forward(spec.replace(shared_mode="none"), w, x)["y"]
    np.testing.assert_allclose(y_blend, 0.5 * y_add, rtol=1e-12, atol=1e-18)
    assert np.abs(y_none).max() > 1e-4 and np.abs(y_add - y_none).max() > 1e-4


def test_blend_coefficients_follow_the_coefficient_head_per_token():
    """Klear PR item 2, second test: the weights are read from the head, per token."""
    spec = SIG_BLEND
    x = np_x(spec, 6)
    w = np_weights(spec)
    c = oracle.forward(spec, w, x)["coef"]
    X = torch.from_numpy(_dec(x))
    logits = X @ torch.from_numpy(_dec(w["coef_w"])).T + torch.from_numpy(_dec(w["coef_b"]))
    np.testing.assert_allclose(c, torch.softmax(logits, dim=-1).numpy(), rtol=1e-13)
    assert np.ptp(c[:, 1]) > 1e-3         # differs between tokens


# --- Klear PR item 3: sigmoid routing, select-only bias, unbiased weights ------
def test_selection_bias_changes_experts_not_weights():
    spec = SIG_BLEND
    T = 6
    x = np_x(spec, T)
    w = np_weights(spec)
    w0 = dict(w, selection_bias=np.zeros_like(w["selection_bias"]))
    base = oracle.forward(spec, w0, x)
    # a constant bias on every expert changes nothing at all
    wc = dict(w, selection_bias=np.full_like(w["selection_bias"], 0.37))
    same = oracle.forward(spec, wc, x)
    assert np.array_equal(same["idx"], base["idx"])
    np.testing.assert_array_equal(same["w"], base["w"])
    np.testing.assert_array_equal(same["y"], base["y"])
    # a large bias on an expert that no token picked forces it into every set
    unused = [e for e in range(spec.num_experts) if not (base["idx"] == e).any()]
    forced = unused[0] if unused else int(np.argmin(np.bincount(base["idx"].ravel(),
                                                                minlength=spec.num_experts)))
    sb = np.zeros_like(w["selection_bias"])
    sb[forced] = 10.0
    out = oracle.forward(spec, dict(w, selection_bias=sb), x)
    assert all(forced in set(r) for r in out["idx"])
    assert not np.array_equal(out["y"], base["y"])
    # the combine weights are the unbiased sigmoid of the chosen set, renormalised
    X = torch.from_numpy(_dec(x))
    p = torch.sigmoid(X @ torch.from_numpy(_dec(w["router_w"])).T).numpy()
    for t in range(T):
        sel = out["idx"][t]
        np.testing.assert_allclose(out["w"][t], p[t, sel] / p[t, sel].sum(), rtol=1e-12)
        biased = (p[t, sel] + sb[sel]) / (p[t, sel] + sb[sel]).sum()
        assert np.abs(out["w"][t] - biased).max() > 1e-2


def test_all_experts_selected_makes_selection_bias_irrelevant():
    """k = E with renormalisation: a select-only bias cannot change the output."""
    spec = SIG_BLEND.replace(top_k=SIG_BLEND.num_experts)
    x = np_x(spec, 4)
    w = np_weights(spec)
    a = oracle.forward(spec, w, x)
    b = oracle.forward(spec, dict(w, selection_bias=np.zeros_like(w["selection_bias"])), x)
    np.testing.assert_allclose(a["y"], b["y"], rtol=1e-13, atol=1e-19)
    np.testing.assert_allclose(a["w"].sum(axis=1), 1.0, rtol=1e-14)


def test_routed_scaling_factor_is_not_applied():
    """Klear PR item 3: 2.5 is declared but not applied; applying it scales routed x2.5."""
    for s in inputs.WORKLOADS.values():
        assert s.routed_scaling_factor == 1.0
    spec = SIG_BLEND.replace(shared_mode="none")
    x = np_x(spec, 5)
    w = np_weights(spec)
    y1 = oracle.forward(spec, w, x)
    y25 = oracle.forward(spec.replace(routed_scaling_factor=2.5), w, x)
    np.testing.assert_allclose(y25["y"], 2.5 * y1["y"], rtol=1e-13)
    np.testing.assert_allclose(y1["w"].sum(axis=1), 1.0, rtol=1e-14)   # norm_topk_prob
    tol = 2e-2 * np.sqrt(np.mean(y1["y"] ** 2))
    assert np.abs(y25["y"] - y1["y"]).max() > 50 * tol


# --- special cases that reduce to textbook / library routines -----------------
def _dense_mlp_torch(X, Wg, Wu, Wd):
    X, Wg, Wu, Wd = (torch.from_numpy(a) for a in (X, Wg, Wu, Wd))
    return (torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T) @ Wd.T).numpy()


def test_single_expert_is_a_dense_swiglu_mlp():
    spec = inputs.TINY_F32.replace(name="t_e1", config_id=110, num_experts=1, top_k=1,
                                   norm_topk_prob=True)
    x = np_x(spec, 9)
    w = np_weights(spec)
    y = oracle.forward(spec, w, x)["y"]
    ref = _dense_mlp_torch(_dec(x), _dec(w["gate_w"][0]), _dec(w["up_w"][0]), _dec(w["down_w"][0]))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-16)


def test_identical_experts_with_renorm_give_the_dense_mlp_for_any_routing():
    spec = SIG_BLEND.replace(shared_mode="none")
    x = np_x(spec, 6)
    w = np_weights(spec)
    for name in ("gate_w", "up_w", "down_w"):
        w[name] = np.ascontiguousarray(np.broadcast_to(w[name][:1], w[name].shape))
    y = oracle.forward(spec, w, x)["y"]
    ref = _dense_mlp_torch(_dec(x), _dec(w["gate_w"][0]), _dec(w["up_w"][0]), _dec(w["down_w"][0]))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-18)


def test_softmax_routing_with_all_experts_is_the_full_soft_mixture():
    spec = inputs.TINY_F32.replace(top_k=inputs.TINY_F32.num_experts)
    x = np_x(spec, 5)
    w = np_weights(spec)
    o = oracle.forward(spec, w, x)
    X = torch.from_numpy(_dec(x))
    p = torch.softmax(X @ torch.from_numpy(_dec(w["router_w"])).T, dim=-1).numpy()
    for t in range(5):
        np.testing.assert_allclose(o["w"][t], p[t, o["idx"][t]], rtol=1e-12)
    np.testing.assert_allclose(o["w"].sum(axis=1), 1.0, rtol=1e-13)
    mix = sum(p[:, e:e + 1] * _dense_mlp_torch(_dec(x), _dec(w["gate_w"][e]), _dec(w["up_w"][e]),
                                               _dec(w["down_w"][e])) for e in range(spec.num_experts))
    np.testing.assert_allclose(o["y"], mix, rtol=1e-11, atol=1e-18)


def test_softmax_topk_weights_are_the_softmax_of_the_selected_logits():
    """libmir-metal ClampedRoutedExperts::forward, router_top_k_unit(top_k)."""
    spec = CLAMPED
    x = np_x(spec, 6, 60.0)
    w = np_weights(spec)
    o = oracle.forward(spec, w, x)
    for t in range(6):
        lg = torch.from_numpy(o["logits"][t, o["idx"][t]])
        np.testing.assert_allclose(o["w"][t], torch.softmax(lg, 0).numpy(), rtol=1e-13)
        assert set(o["idx"][t]) == set(torch.topk(torch.from_numpy(o["logits"][t]),
                                                  spec.top_k).indices.tolist())
    k1 = oracle.forward(spec.replace(top_k=1), w, x)
    assert np.all(k1["w"] == 1.0)


def test_latent_with_identity_projections_is_moe_then_rmsnorm():
    """ferrox latent_moe.rs flow with down_proj = up_proj = I and latent = hidden."""
    spec = LATENT.replace(latent_dim=LATENT.hidden, shared_mode="none", rms_eps=1e-6,
                          act_dtype="f32", weight_format="f32", name="t_lat_id", config_id=111)
    x = np_x(spec, 5)
    w = np_weights(spec)
    eye = np.eye(spec.hidden, dtype=np.float32)
    w["latent_down_w"], w["latent_up_w"] = eye.copy(), eye.copy()
    y = oracle.forward(spec, w, x)["y"]
    plain = spec.replace(latent_dim=0, latent_use_norm=False)
    z = oracle.forward(plain, w, x)["y"]
    ref = torch.nn.functional.rms_norm(torch.from_numpy(z), (spec.hidden,),
                                       weight=torch.from_numpy(_dec(w["latent_norm_w"])),
                                       eps=spec.rms_eps).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_latent_norm_removes_the_scale_of_the_routed_branch():
    """RMSNorm after the combine: scaling every down plane by a > 0 cancels (eps -> 0);
    without the norm the output moves and stays finite (ferrox second test)."""
    spec = LATENT.replace(rms_eps=1e-30)
    x = np_x(spec, 4)
    w = np_weights(spec)
    wa = dict(w)
    wa["down_w"] = to_bf16_bits(_dec(w["down_w"]) * 4.0)      # x4 is exact in bf16
    np.testing.assert_allclose(oracle.forward(spec, wa, x)["y"], oracle.forward(spec, w, x)["y"],
                               rtol=1e-11, atol=1e-17)
    nn = spec.replace(latent_use_norm=False)
    a, b = oracle.forward(nn, wa, x)["y"], oracle.forward(nn, w, x)["y"]
    assert np.all(np.isfinite(a)) and np.abs(a - b).max() > 1e-6


def test_page_example_without_routed_norm_is_finite_and_differs():
    """ferrox latent_moe.rs tests: without_routed_norm_output_still_finite_and_differs,
    on the page's own weights (SwiGLU in place of the undefined situ)."""
    fx = json.load(open(os.path.join(GOLDEN, "latent_moe_kimi_example.json")))
    d = fx["dims"]
    spec = inputs.MoeSpec(name="kimi_example", config_id=0, hidden=d["hidden"],
                          num_experts=d["num_experts"], top_k=d["top_k"],
                          intermediate=d["intermediate"], scoring="sigmoid",
                          has_selection_bias=True, norm_topk_prob=True, act_dtype="f32",
                          weight_format="f32", shared_mode="add",
                          shared_intermediate=d["shared_intermediate"], latent_dim=d["latent"],
                          latent_use_norm=True, rms_eps=d["rms_eps"])
    f = lambda k, *shape: np.asarray(fx[k], dtype=np.float32).reshape(shape)
    H, L, I, E, Is = 6, 4, 3, 4, 3
    w = {"router_w": f("router_weight", E, H), "selection_bias": f("bias", E),
         "latent_down_w": f("down_proj", L, H), "latent_up_w": f("up_proj", H, L),
         "latent_norm_w": f("routed_norm_w", L),
         "gate_w": np.stack([f(f"e{e}_w1", I, L) for e in range(E)]),
         "down_w": np.stack([f(f"e{e}_w2", L, I) for e in range(E)]),
         "up_w": np.stack([f(f"e{e}_w3", I, L) for e in range(E)]),
         "shared_gate_w": f("shared_w1", Is, H), "shared_down_w": f("shared_w2", H, Is),
         "shared_up_w": f("shared_w3", Is, H)}
    x = f("hidden", 1, H)
    with_norm = oracle.forward(spec, w, x)["y"][0]
    without = oracle.forward(spec.replace(latent_use_norm=False), w, x)["y"][0]
    assert np.all(np.isfinite(without))
    assert abs(without[0] - with_norm[0]) > 1e-6
    b = bruteforce.forward(spec, w, x)["y"][0]
    np.testing.assert_allclose(with_norm, b, rtol=1e-12)


def test_batch_equals_tokens_one_at_a_time():
    """Klear PR validation, causality check: a token's output does not depend on the
    other tokens in the batch (exact in the oracle)."""
    spec = Q4
    x = np_x(spec, 6)
    w = np_weights(spec)
    full = oracle.forward(spec, w, x)
    for t in range(6):
        one = oracle.forward(spec, w, np.ascontiguousarray(x[t:t + 1]))
        np.testing.assert_array_equal(one["y"][0], full["y"][t])
        np.testing.assert_array_equal(one["idx"][0], full["idx"][t])
    sub = oracle.forward(spec, w, x, tokens=[4, 1])
    np.testing.assert_array_equal(sub["y"], full["y"][[4, 1]])


def test_forward_with_indices_reproduces_the_routed_choice():
    spec = SIG_BLEND
    x = np_x(spec, 4)
    w = np_weights(spec)
    full = oracle.forward(spec, w, x)
    for t in range(4):
        y, wt = oracle.forward_with_indices(spec, w, x, t, full["idx"][t])
        np.testing.assert_array_equal(y, full["y"][t])
        np.testing.assert_array_equal(wt, full["w"][t])
    # another set gives another output
    other = [e for e in range(spec.num_experts) if e not in full["idx"][0]][:spec.top_k]
    y, _ = oracle.forward_with_indices(spec, w, x, 0, other)
    assert np.abs(y - full["y"][0]).max() > 1e-6


def test_exact_key_ties_go_to_the_lower_expert_index():
    spec = ROUTER_BIAS.replace(has_router_bias=False, norm_topk_prob=False)
    w = np_weights(spec)
    rw = np.zeros_like(w["router_w"])
    v = np.linspace(0.5, 1.5, spec.hidden).astype(np.float32)
    rw[2] = v
    rw[5] = v
    w["router_w"] = rw
    x = np.abs(np_x(spec, 3)) + np.float32(0.1)      # x . v > 0: experts 2 and 5 lead, tied
    o = oracle.forward(spec, w, x.astype(np.float32))
    for t in range(3):
        assert list(o["idx"][t]) == [2, 5, 0]         # then the tied zeros: lowest index first
    s = oracle.forward(spec.replace(scoring="sigmoid"), w, x.astype(np.float32))
    assert all(list(r) == [2, 5, 0] for r in s["idx"])


# --- activations ----------------------------------------------------------------
def test_swiglu_is_silu_gate_times_up():
    for g, v in [(-3.0, 0.7), (0.0, 5.0), (1.25, -2.0), (9.0, 1.0)]:
        ref = float(torch.nn.functional.silu(torch.tensor(g, dtype=torch.float64))) * v
        assert oracle.activation("swiglu", g, v) == pytest.approx(ref, rel=1e-15, abs=1e-300)


def test_clamped_swiglu_closed_forms():
    act = lambda g, v: oracle.activation("swiglu_clamped", g, v, 7.0, 1.702)
    for v in (-3.0, 0.5, 4.0):
        assert act(7.0, v) == act(11.0, v) == act(1e6, v)          # constant for gate >= 7
    for g in (-2.0, 0.3, 5.0):
        assert act(g, 7.0) == act(g, 50.0) == pytest.approx(8.0 * act(g, 0.0), rel=1e-15)
        assert act(g, -7.0) == act(g, -50.0) == pytest.approx(-6.0 * act(g, 0.0), rel=1e-15)
        assert act(g, -1.0) == 0.0
    assert act(0.0, 3.0) == 0.0
    # below the clamp it is g * sigmoid(1.702 g) * (v + 1): check against torch
    g = torch.tensor(2.5, dtype=torch.float64)
    assert act(2.5, 1.5) == pytest.approx(float(g * torch.sigmoid(1.702 * g)) * 2.5, rel=1e-15)


# --- 4-bit affine ----------------------------------------------------------------
def test_q4_dequant_of_hand_set_words_is_exact():
    """mlxcel issue #974: affine mode, weight + per-group scales + biases."""
    q = np.array([[0x76543210, 0xFEDCBA98]], dtype=np.uint32)     # codes 0..15 in order
    s = to_bf16_bits(np.array([[0.5]]))
    z = to_bf16_bits(np.array([[-1.0]]))
    vals = [oracle.dequant_q4(q, s, z, 16, 16, 0, c) for c in range(16)]
    assert vals == [0.5 * c - 1.0 for c in range(16)]
    # two groups of 8 with their own scale/bias
    s2 = to_bf16_bits(np.array([[2.0, 0.25]]))
    z2 = to_bf16_bits(np.array([[0.0, 3.0]]))
    vals = [oracle.dequant_q4(q, s2, z2, 16, 8, 0, c) for c in range(16)]
    assert vals == [2.0 * c for c in range(8)] + [0.25 * c + 3.0 for c in range(8, 16)]


def test_q4_planes_match_the_bruteforce_unpacking_and_are_near_the_drawn_weights():
    spec = Q4
    w = np_weights(spec)
    deq = bruteforce._dequant(w["gate_w"], w["gate_s"], w["gate_z"], spec.group_size)
    for (e, r, c) in [(0, 0, 0), (1, 5, 63), (3, 63, 127), (2, 17, 64)]:
        assert oracle.dequant_q4(w["gate_w"].reshape(-1, spec.hidden // 8),
                                 w["gate_s"].reshape(-1, spec.hidden // 64),
                                 w["gate_z"].reshape(-1, spec.hidden // 64), spec.hidden, 64,
                                 e * spec.intermediate + r, c) == deq[e, r, c]
    assert np.abs(deq).max() < 0.2 and deq.std() == pytest.approx(0.02, rel=0.1)


# --- MXFP4 (OCP Microscaling Formats v1.0) -----------------------------------------
# The FP4 E2M1 value table of the specification, by code 0..15.
SPEC_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_mxfp4_codes_decode_to_the_spec_table_times_the_block_scale():
    q = np.array([[0x76543210, 0xFEDCBA98, 0x76543210, 0xFEDCBA98]], dtype=np.uint32)  # codes 0..15, twice
    for sbyte in (127, 120, 130, 1, 254):
        s = np.array([[sbyte]], dtype=np.uint8)
        vals = [oracle.dequant_mxfp4(q, s, 32, 0, c) for c in range(32)]
        assert vals == [v * 2.0 ** (sbyte - 127) for v in SPEC_E2M1 * 2]
    assert math.isnan(oracle.dequant_mxfp4(q, np.array([[255]], dtype=np.uint8), 32, 0, 3))  # NaN scale
    # two blocks of 32 with their own scales, element j at bits 4 * (j mod 8) of word j / 8
    q2 = np.array([[0x00000001] + [0] * 3 + [0x60000000] + [0] * 3], dtype=np.uint32)
    s2 = np.array([[127, 125]], dtype=np.uint8)
    assert oracle.dequant_mxfp4(q2, s2, 64, 0, 0) == 0.5
    assert oracle.dequant_mxfp4(q2, s2, 64, 0, 39) == 4.0 * 0.25   # code 6 = 4.0, block scale 2^-2


def test_mxfp4_encoder_keeps_representable_values_and_matches_bruteforce_unpacking():
    vals = torch.tensor(SPEC_E2M1[:8] + [-v for v in SPEC_E2M1[1:8]] + [6.0] * 17) * 2.0 ** -9
    q, s = inputs.quantize_mxfp4(vals.reshape(1, 32).float())
    qn, sn = inputs.to_numpy_storage(q), inputs.to_numpy_storage(s)
    assert [oracle.dequant_mxfp4(qn, sn, 32, 0, c) for c in range(32)] == vals.double().tolist()
    w = np_weights(MXFP4)
    deq = bruteforce._dequant_mxfp4(w["gate_w"], w["gate_s"])
    for (e, r, c) in [(0, 0, 0), (1, 5, 63), (4, 63, 127), (2, 17, 64)]:
        assert oracle.dequant_mxfp4(w["gate_w"].reshape(-1, MXFP4.hidden // 8),
                                    w["gate_s"].reshape(-1, MXFP4.hidden // 32), MXFP4.hidden,
                                    e * MXFP4.intermediate + r, c) == deq[e, r, c]
    assert np.abs(deq).max() < 0.2 and deq.std() == pytest.approx(0.02, rel=0.15)


def test_mxfp4_block_equals_the_same_weights_stored_in_bf16():
    """Every MXFP4 weight (at most two significant bits times a power of two) is exact in bf16:
    the block evaluated on the packed planes equals the block on those values stored as bf16."""
    w = np_weights(MXFP4)
    x = np_x(MXFP4, 6, 30.0)
    spec_bf = MXFP4.replace(name="t_mxfp4_as_bf16", weight_format="bf16")
    wb = dict(w)
    for name in ("gate_w", "up_w", "down_w"):
        deq = bruteforce._dequant_mxfp4(w[name], w[name[:-2] + "_s"])
        wb[name] = to_bf16_bits(deq)
        del wb[name[:-2] + "_s"]
    a = oracle.forward(MXFP4, w, x)
    b = oracle.forward(spec_bf, wb, x)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_array_equal(a["y"], b["y"])


@pytest.mark.parametrize("spec", [MXFP4_NATIVE, Q4_INTERLEAVED], ids=lambda s: s.name)
def test_interleaved_4bit_block_equals_the_split_block_on_the_same_rows(spec):
    """The native layout's single gate_up plane (libmir-metal ExpertLayout::Native), read as
    row 2i gate and 2i + 1 up with the companions and bias in the same row order, is the split
    layout of its even and odd rows: the two evaluations agree exactly."""
    w = np_weights(spec)
    x = np_x(spec, 7, 30.0)
    split = spec.replace(name=spec.name + "_split", gate_up_interleaved=False)
    ws = {k: v for k, v in w.items() if not k.startswith("gate_up")}
    for comp in ("_w", "_s", "_z", "_b"):
        if "gate_up" + comp in w:
            plane = w["gate_up" + comp]
            ws["gate" + comp], ws["up" + comp] = plane[:, 0::2].copy(), plane[:, 1::2].copy()
    a = oracle.forward(spec, w, x)
    b = oracle.forward(split, ws, x)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_array_equal(a["y"], b["y"])
    # and a swapped row order (up rows first) is a different block
    wswap = dict(w)
    g = w["gate_up_w"]
    wswap["gate_up_w"] = np.stack([g[:, 1::2], g[:, 0::2]], axis=2).reshape(g.shape).copy()
    assert not np.array_equal(oracle.forward(spec, wswap, x)["y"], a["y"])


# --- 4-bit dense planes (router, shared expert, latent projections) --------------
def _exact_q4(rows, cols, group, rng):
    """A 4-bit affine plane whose every weight is exact in bf16: scale 2^-6, bias -8 * 2^-6,
    so weight = (q - 8) / 64 with q in [0, 15]. Returns (words, scales, biases, values)."""
    q = rng.integers(0, 16, size=(rows, cols)).astype(np.uint32)
    words = np.zeros((rows, cols // 8), dtype=np.uint32)
    for j in range(8):
        words |= q[:, j::8] << np.uint32(4 * j)
    s = np.full((rows, cols // group), 2.0 ** -6, dtype=np.float32)
    z = np.full((rows, cols // group), -8 * 2.0 ** -6, dtype=np.float32)
    return words, to_bf16_bits(s), to_bf16_bits(z), (q.astype(np.float64) - 8) / 64


def test_dense_q4_block_equals_the_bf16_block_on_the_same_exact_values():
    """With every dense weight exact in bf16, the block reading the 4-bit dense planes equals
    the block reading those values stored as bf16, exactly."""
    spec = DENSE_Q4
    rng = np.random.default_rng(3)
    w = np_weights(spec)
    shapes = {"router_w": (spec.num_experts, spec.hidden),
              "shared_gate_w": (spec.shared_intermediate, spec.hidden),
              "shared_up_w": (spec.shared_intermediate, spec.hidden),
              "shared_down_w": (spec.hidden, spec.shared_intermediate),
              "latent_down_w": (spec.latent_dim, spec.hidden),
              "latent_up_w": (spec.hidden, spec.latent_dim)}
    wq, wb = dict(w), dict(w)
    for name, (r, c) in shapes.items():
        words, s, z, vals = _exact_q4(r, c, spec.dense_group_size, rng)
        wq[name], wq[name[:-2] + "_s"], wq[name[:-2] + "_z"] = words, s, z
        wb[name] = to_bf16_bits(vals)
        for comp in ("_s", "_z"):
            wb.pop(name[:-2] + comp, None)
    x = np_x(spec, 6)
    a = oracle.forward(spec, wq, x)
    b = oracle.forward(spec.replace(name="t_dense_as_bf16", dense_format="act"), wb, x)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_array_equal(a["y"], b["y"])
    assert np.abs(a["y"]).max() > 0


def test_dense_q4_planes_change_the_output_against_the_unquantised_draw():
    """The 4-bit dense planes are a different block from the drawn bf16 planes (they are read,
    not ignored), yet close to it: the quantisation error of the dense parts is small."""
    spec = DENSE_Q4
    x = np_x(spec, 5)
    yq = oracle.forward(spec, np_weights(spec), x)["y"]
    y16 = oracle.forward(spec.replace(dense_format="act"), np_weights(spec.replace(dense_format="act")), x)["y"]
    assert not np.array_equal(yq, y16)
    assert np.abs(yq - y16).max() < 0.5 * np.abs(y16).max()


# --- permutation -----------------------------------------------------------------
def test_permutation_is_the_stable_sort_of_slots_by_expert():
    rng = np.random.default_rng(0)
    for T, k, E in [(1, 8, 256), (37, 4, 16), (500, 8, 64), (3, 2, 8)]:
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        off, ss, pos = oracle.permute(idx, E)
        flat = idx.ravel()
        np.testing.assert_array_equal(ss, np.argsort(flat, kind="stable"))
        np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        np.testing.assert_array_equal(pos[ss], np.arange(T * k))
        assert off[-1] == T * k
