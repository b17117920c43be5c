"""The seeded synthetic inputs: deterministic, distinct per workload and size, and drawn
from the stated distributions (x ~ N(0, 1); weights ~ N(0, 0.02); select-only bias
~ N(0, 0.1); RMSNorm gamma = 1 + N(0, 0.1))."""
import numpy as np
import pytest
import torch

from sparse_moe_ffn_gemv_b200 import inputs
from tiny_specs import LATENT, MXFP4_NATIVE, Q4, SIG_BLEND


@pytest.mark.parametrize("spec", [SIG_BLEND, Q4, LATENT, MXFP4_NATIVE], ids=lambda s: s.name)
def test_generation_is_deterministic(spec):
    a, b = inputs.make_weights(spec, threads=1), inputs.make_weights(spec, threads=3)
    assert a.keys() == b.keys()
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(inputs.make_x(spec, 5), inputs.make_x(spec, 5))


def test_inputs_differ_across_sizes_and_workloads():
    assert not torch.equal(inputs.make_x(SIG_BLEND, 5)[:1], inputs.make_x(SIG_BLEND, 6)[:1])
    other = SIG_BLEND.replace(config_id=SIG_BLEND.config_id + 1)
    assert not torch.equal(inputs.make_weights(SIG_BLEND)["router_w"], inputs.make_weights(other)["router_w"])


def test_draws_follow_the_stated_distributions():
    spec = inputs.KLEAR_BF16
    x = inputs.make_x(spec, 512).float()
    assert abs(float(x.mean())) < 0.01 and float(x.std()) == pytest.approx(1.0, rel=0.01)
    w = inputs.make_weights(LATENT.replace(hidden=512, latent_dim=256, num_experts=64, intermediate=32))
    r = w["router_w"].float()
    assert float(r.std()) == pytest.approx(0.02, rel=0.02) and abs(float(r.mean())) < 1e-3
    sb = w["selection_bias"].float()
    assert sb.dtype == torch.float32 and float(sb.std()) == pytest.approx(0.1, rel=0.25)
    gam = w["latent_norm_w"].float()
    assert float(gam.mean()) == pytest.approx(1.0, abs=0.03) and float(gam.std()) == pytest.approx(0.1, rel=0.2)


def test_4bit_codes_stay_in_range_and_scales_are_positive():
    w = inputs.make_weights(Q4)
    codes = inputs.to_numpy_storage(w["gate_w"])
    nib = (codes[..., None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF
    assert nib.min() == 0 and nib.max() == 15          # min/max quantiser: both ends used
    assert (w["gate_s"].float() > 0).all()
    wm = inputs.make_weights(MXFP4_NATIVE)
    assert wm["gate_up_w"].shape == (MXFP4_NATIVE.num_experts, 2 * MXFP4_NATIVE.intermediate,
                                     MXFP4_NATIVE.hidden // 8)
    assert wm["gate_up_s"].dtype == torch.uint8
    assert wm["gate_up_s"].shape == (MXFP4_NATIVE.num_experts, 2 * MXFP4_NATIVE.intermediate,
                                     MXFP4_NATIVE.hidden // 32)
