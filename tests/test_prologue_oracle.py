"""Pins of the prologue oracle (oracle/prologue.py) against closed forms,
brute force and invariants -- no GPU.

Each pin is chosen so that a plausible slip in the oracle fails it: the tap
order of the convolution (identity and one-hot taps, brute force), the ring
slot of a position (pos0 not a multiple of 4, streaming in two parts), the
activation (closed forms), the L2 norm (unit norms), and the gate bound.
"""
import math

import numpy as np
import pytest

from oracle import prologue as P

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _inputs(B=2, T=9, H=2, dk=4, dv=3, seed=0, gate="scalar"):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk))
    v = rng.normal(size=(B, T, H, dv))
    g = rng.normal(size=(B, T, H) if gate == "scalar" else (B, T, H, dk)) * 3
    beta = rng.normal(size=(B, T, H))
    w = rng.normal(size=(H, 2 * dk + dv, 4))
    return q, k, v, g, beta, w


def test_identity_taps_and_one_hot_taps():
    q, k, v, g, beta, w = _inputs()
    C = w.shape[1]
    w_id = np.zeros_like(w)
    w_id[..., 3] = 1.0                       # current token only
    qo, ko, vo, _, _, _ = P.prologue(q, k, v, g, beta, w_id, activation="none")
    np.testing.assert_array_equal(vo, v)
    np.testing.assert_allclose(qo, q / np.sqrt((q * q).sum(-1, keepdims=True) + 1e-6), rtol=1e-15)
    # tap 0 alone picks the input three tokens back (zero history before t = 3)
    w0 = np.zeros_like(w)
    w0[..., 0] = 1.0
    _, _, vo, _, _, _ = P.prologue(q, k, v, g, beta, w0, activation="none")
    np.testing.assert_array_equal(vo[:, 3:], v[:, :-3])
    np.testing.assert_array_equal(vo[:, :3], 0.0)
    assert C == 2 * q.shape[-1] + v.shape[-1]


def test_convolution_against_brute_force_loops():
    q, k, v, g, beta, w = _inputs(seed=1)
    B, T, H, dk = q.shape
    x = np.concatenate([q, k, v], -1)
    rng = np.random.default_rng(5)
    ring = rng.normal(size=(B, H, 4, x.shape[-1]))
    pos0 = np.array([6, 1])
    _, _, vo, _, _, _ = P.prologue(q, k, v, g, beta, w, ring, pos0, activation="none")
    for b in range(B):
        for t in range(T):
            for h in range(H):
                for c in range(2 * dk, x.shape[-1]):
                    acc = 0.0
                    for j in range(4):
                        tt = t - 3 + j
                        if tt >= 0:
                            val = x[b, tt, h, c]
                        else:
                            p = pos0[b] + tt
                            val = ring[b, h, p % 4, c] if p >= 0 else 0.0
                        acc += w[h, c, j] * val
                    assert math.isclose(vo[b, t, h, c - 2 * dk], acc, rel_tol=1e-12, abs_tol=1e-12)


def test_streaming_in_two_parts_equals_one_pass():
    q, k, v, g, beta, w = _inputs(T=11, seed=2, gate="channel")
    B, T, H, dk = q.shape
    C = w.shape[1]
    ring0 = np.random.default_rng(3).normal(size=(B, H, 4, C))
    pos0 = np.array([5, 2])
    full = P.prologue(q, k, v, g, beta, w, ring0, pos0)
    T1 = 4
    a = P.prologue(q[:, :T1], k[:, :T1], v[:, :T1], g[:, :T1], beta[:, :T1], w, ring0, pos0)
    bpart = P.prologue(q[:, T1:], k[:, T1:], v[:, T1:], g[:, T1:], beta[:, T1:], w, a[5], pos0 + T1)
    for i in range(5):
        np.testing.assert_allclose(np.concatenate([a[i], bpart[i]], axis=1), full[i], rtol=1e-13,
                                   atol=1e-14)
    np.testing.assert_allclose(bpart[5], full[5])


def test_ring_after_keeps_untouched_slots_for_short_inputs():
    q, k, v, g, beta, w = _inputs(T=2, seed=4)
    B, T, H, dk = q.shape
    C = w.shape[1]
    ring = np.random.default_rng(7).normal(size=(B, H, 4, C))
    pos0 = np.array([3, 8])
    ring_out = P.prologue(q, k, v, g, beta, w, ring, pos0)[5]
    x = np.concatenate([q, k, v], -1)
    for b in range(B):
        written = {(pos0[b] + t) % 4: t for t in range(T)}
        for s in range(4):
            expect = x[b, written[s]] if s in written else ring[b, :, s]
            np.testing.assert_array_equal(ring_out[b, :, s], expect)


def test_activation_gate_and_norm_closed_forms():
    assert P.silu(np.array(0.0)) == 0.0
    assert math.isclose(float(P.silu(np.array(2.0))), 2.0 / (1.0 + math.exp(-2.0)), rel_tol=1e-15)
    assert float(P.sigmoid(np.array(0.0))) == 0.5
    assert math.isclose(float(P.softplus(np.array(0.0))), math.log(2.0), rel_tol=1e-15)
    assert float(P.softplus(np.array(80.0))) == 80.0
    q, k, v, _, beta, w = _inputs(seed=6)
    g = np.array([100.0, 3.0, 0.0, -3.0, -100.0]).reshape(1, 5, 1).repeat(2, 0).repeat(2, 2)
    g = np.concatenate([g, np.zeros((2, 4, 2))], axis=1)
    _, _, _, go, bo, _ = P.prologue(q, k, v, g, beta, w)
    assert go[0, 0, 0] == -5.0                               # bound
    assert math.isclose(go[0, 1, 0], -math.log1p(math.exp(3.0)), rel_tol=1e-15)
    assert math.isclose(go[0, 2, 0], -math.log(2.0), rel_tol=1e-15)
    assert -1e-40 < go[0, 4, 0] <= 0.0                       # -softplus(-100), tiny
    assert (go <= 0).all() and (go >= -5).all()
    np.testing.assert_allclose(bo, 1.0 / (1.0 + np.exp(-beta)), rtol=1e-15)
    qo, ko, _, _, _, _ = P.prologue(q, k, v, g, beta, w)
    for t in (qo, ko):
        n2 = (t * t).sum(-1)
        assert (n2 <= 1.0).all() and (n2 > 0.99).all()
