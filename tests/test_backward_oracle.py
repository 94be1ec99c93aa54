"""Pins of the gradient oracle (oracle/backward.py) -- CPU only.

The gradients are pinned to the forward recurrence by central finite
differences of the C forward oracle (oracle/gdn_oracle.c, separate code),
for every input and both gate modes, with an initial state and a gradient
arriving at the final state; a one-token closed form pins the algebra again
by hand.  A dropped term, a wrong sign or a transposed product in any line
of the reverse sweep moves some gradient far outside the finite-difference
error (~1e-9 here).
"""
import numpy as np
import pytest

import oracle
from oracle import backward as BW


def _case(per_channel, seed, B=1, T=5, H=2, dk=3, dv=2):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk)) / np.sqrt(dk)
    v = rng.normal(size=(B, T, H, dv))
    g = -np.abs(rng.normal(size=(B, T, H, dk) if per_channel else (B, T, H))) * 0.5
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H))))
    s0 = rng.normal(size=(B, H, dk, dv)) * 0.3
    do = rng.normal(size=(B, T, H, dv))
    dsT = rng.normal(size=(B, H, dk, dv))
    return dict(q=q, k=k, v=v, g=g, beta=beta, s0=s0), do, dsT


def _loss(x, do, dsT, per_channel):
    o, sT = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=per_channel,
                       threads=1)
    return float(np.sum(do * o) + np.sum(dsT * sT))


@pytest.mark.parametrize("per_channel", [True, False])
def test_forward_matches_c_oracle(per_channel):
    x, _, _ = _case(per_channel, 1, B=2, T=7, H=3, dk=4, dv=5)
    o1, s1 = oracle.run(**x, per_channel=per_channel, threads=1)
    o2, s2, _ = BW.forward(**x, per_channel=per_channel)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s1, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("per_channel", [True, False])
def test_gradients_match_central_differences(per_channel):
    x, do, dsT = _case(per_channel, 2)
    grads = BW.backward(**x, d_out=do, d_state=dsT, per_channel=per_channel)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "s0": "ds0"}
    h = 1e-6
    for name, gname in names.items():
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = {n: a.copy() for n, a in x.items()}
            xm = {n: a.copy() for n, a in x.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            fd[idx] = (_loss(xp, do, dsT, per_channel) - _loss(xm, do, dsT, per_channel)) / (2 * h)
        err = np.max(np.abs(grads[gname] - fd))
        assert err <= 1e-7 * max(1.0, np.max(np.abs(fd))), (gname, err)


def test_one_token_closed_form():
    """T = 1, S0 = 0: o = beta (k . q) v, so dq = beta (v . do) k,
    dk = beta (v . do) q, dv = beta (k . q) do, dbeta = (k . q)(v . do), and
    the gate has no effect (dg = 0)."""
    rng = np.random.default_rng(3)
    q, k = rng.normal(size=(1, 1, 1, 4)), rng.normal(size=(1, 1, 1, 4))
    v, do = rng.normal(size=(1, 1, 1, 3)), rng.normal(size=(1, 1, 1, 3))
    g = np.array([[[-0.7]]])
    beta = np.array([[[0.6]]])
    r = BW.backward(q, k, v, g, beta, None, do, per_channel=False)
    kq = float(np.sum(k * q))
    vdo = float(np.sum(v * do))
    np.testing.assert_allclose(r["dq"][0, 0, 0], 0.6 * vdo * k[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(r["dk"][0, 0, 0], 0.6 * vdo * q[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(r["dv"][0, 0, 0], 0.6 * kq * do[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(r["dbeta"][0, 0, 0], kq * vdo, rtol=1e-14)
    assert r["dg"][0, 0, 0] == 0.0
    np.testing.assert_allclose(r["ds0"][0, 0], np.exp(-0.7) * (
        np.outer(q[0, 0, 0], do[0, 0, 0]) - 0.6 * np.outer(k[0, 0, 0], k[0, 0, 0]) @ np.outer(q[0, 0, 0], do[0, 0, 0])),
        rtol=1e-13, atol=1e-15)


def test_scalar_gate_gradient_is_the_sum_of_equal_channel_gradients():
    """A scalar gate is a per-channel gate with all channels equal, so its
    gradient is the sum over channels of the per-channel gradient."""
    x, do, dsT = _case(False, 4, B=2, T=6, H=2, dk=4, dv=3)
    xc = dict(x, g=np.repeat(x["g"][..., None], 4, axis=-1))
    rs = BW.backward(**x, d_out=do, d_state=dsT, per_channel=False)
    rc = BW.backward(**xc, d_out=do, d_state=dsT, per_channel=True)
    np.testing.assert_allclose(rs["dg"], rc["dg"].sum(-1), rtol=1e-12, atol=1e-14)
    for n in ("dq", "dk", "dv", "dbeta", "ds0"):
        np.testing.assert_allclose(rs[n], rc[n], rtol=1e-12, atol=1e-14)
