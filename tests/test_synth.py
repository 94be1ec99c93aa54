"""The seeded input recipe (CPU only)."""
import torch

from synth import CONFIGS, config_inputs, decode_inputs, prefill_inputs


def test_prefill_recipe_properties():
    x = prefill_inputs(2, 100, 3, 64, 32, gate="channel", io=torch.bfloat16, s0_std=0.1,
                       g_zero_frac=0.1, seed=5)
    assert x["q"].dtype == torch.bfloat16 and x["q"].shape == (2, 100, 3, 64)
    assert x["v"].shape == (2, 100, 3, 32)
    assert x["g"].shape == (2, 100, 3, 64) and x["g"].dtype == torch.float32
    assert x["beta"].shape == (2, 100, 3)
    assert x["s0"].shape == (2, 3, 64, 32)
    n = x["k"].float().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=2e-2)
    assert float(x["g"].max()) <= 0.0 and float(x["g"].min()) >= -5.0
    assert 0.0 < float(x["beta"].min()) and float(x["beta"].max()) < 1.0
    zero_rows = (x["g"] == 0).all(dim=-1).float().mean()
    assert 0.05 < float(zero_rows) < 0.15
    assert abs(float(x["s0"].std()) - 0.1) < 0.01


def test_determinism_and_seed_sensitivity():
    a = prefill_inputs(1, 10, 2, 16, 16, seed=1)
    b = prefill_inputs(1, 10, 2, 16, 16, seed=1)
    c = prefill_inputs(1, 10, 2, 16, 16, seed=2)
    for key in ("q", "k", "v", "g", "beta"):
        assert torch.equal(a[key], b[key])
    assert not torch.equal(a["q"], c["q"])


def test_sliced_draw_spans_slices():
    import synth
    x = prefill_inputs(1, synth.SLICE_TOKENS + 17, 1, 8, 8, seed=3)
    assert x["q"].shape[1] == synth.SLICE_TOKENS + 17
    # two slices are different draws
    assert not torch.equal(x["q"][0, :17], x["q"][0, synth.SLICE_TOKENS:])


def test_decode_recipe():
    x = decode_inputs(3, 2, 16, 8, 5, gate="channel", seed=4)
    assert x["q"].shape == (5, 3, 2, 16) and x["g"].shape == (5, 3, 2, 16)
    assert x["s0"].shape == (3, 2, 16, 8)


def test_configs_reduced_overrides():
    cfg = CONFIGS[3]
    x = config_inputs(cfg, T=64, B=1, H=2)
    assert x["q"].shape == (1, 64, 2, 128) and x["g"].shape == (1, 64, 2)
    assert x["s0"] is not None
