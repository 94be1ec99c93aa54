"""The fp64 oracle checked against what the formula and mathematics fix (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.run)


def test_head_selection_matches_full_run():
    q, k, v, g, beta, S0 = pins.random_case(7, B=3, H=2, T=5, per_channel=True)
    out, sT = oracle.run(q, k, v, g, beta, S0, per_channel=True)
    o2, s2 = oracle.run(q, k, v, g, beta, S0, per_channel=True, heads=[1, 4])
    for bh in (1, 4):
        b, h = divmod(bh, 2)
        np.testing.assert_array_equal(o2[b, :, h], out[b, :, h])
        np.testing.assert_array_equal(s2[b, h], sT[b, h])
    assert np.isnan(o2[0, :, 0]).all()


def test_run_steps_is_a_relayout():
    q, k, v, g, beta, S0 = pins.random_case(8, B=2, H=3, T=4, per_channel=False)
    out, sT = oracle.run(q, k, v, g, beta, S0, per_channel=False)
    sw = lambda x: np.swapaxes(x, 0, 1)  # noqa: E731
    o_s, s_s = oracle.run_steps(sw(q), sw(k), sw(v), sw(g), sw(beta), S0, per_channel=False)
    np.testing.assert_array_equal(sw(o_s), out)
    np.testing.assert_array_equal(s_s, sT)


def test_oracle_threads_do_not_change_results():
    q, k, v, g, beta, S0 = pins.random_case(9, B=4, H=4, T=6, per_channel=True)
    a = oracle.run(q, k, v, g, beta, S0, per_channel=True, threads=1)
    b = oracle.run(q, k, v, g, beta, S0, per_channel=True, threads=4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_realistic_size_against_transition_form():
    """dk=dv=16 with the synthetic recipe; still small enough for the dense form."""
    from oracle import dense
    from synth import prefill_inputs
    import torch
    x = prefill_inputs(1, 24, 2, 16, 16, gate="channel", io=torch.float32, s0_std=0.1, seed=3)
    out, sT = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=True)
    f = lambda t: t.double().numpy()  # noqa: E731
    o_d, s_d = dense.transition_form(f(x["q"]), f(x["k"]), f(x["v"]), f(x["g"]), f(x["beta"]),
                                     f(x["s0"]), per_channel=True)
    pins.close(out, o_d, what="outputs")
    pins.close(sT, s_d, what="state")
