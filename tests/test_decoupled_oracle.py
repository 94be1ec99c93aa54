"""Pins of the decoupled erase / write oracle (oracle/decoupled.py) -- CPU.

The form itself is a reading (the pages give no formula: parity unpinned);
these pins fix its arithmetic against independent code and closed forms.
"""
import numpy as np
import pytest

import oracle
from oracle import decoupled as DC


def _case(per_channel, seed, B=2, T=9, H=2, dk=5, dv=4):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(B, T, H, dv))
    g = -np.abs(rng.normal(size=(B, T, H, dk) if per_channel else (B, T, H)))
    be = rng.uniform(0, 1, size=(B, T, H))
    bw = rng.uniform(0, 1, size=(B, T, H))
    s0 = rng.normal(size=(B, H, dk, dv)) * 0.3
    return q, k, v, g, be, bw, s0


@pytest.mark.parametrize("per_channel", [True, False])
def test_equal_gates_reproduce_the_coupled_oracle(per_channel):
    q, k, v, g, be, _, s0 = _case(per_channel, 1)
    o1, s1 = DC.run(q, k, v, g, be, be, s0, per_channel=per_channel)
    o2, s2 = oracle.run(q, k, v, g, be, s0, per_channel=per_channel, threads=1)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("per_channel", [True, False])
def test_no_erase_is_gated_linear_attention(per_channel):
    """be = 0: S_t = Diag(a_t) S_{t-1} + bw_t k_t v_t^T, so
    o_t = S0^T (P_t (.) q_t) + sum_{s<=t} bw_s (q_t^T Diag(P_t / P_s) k_s) v_s
    with P_t = prod_{r<=t} a_r."""
    q, k, v, g, _, bw, s0 = _case(per_channel, 2)
    be = np.zeros_like(bw)
    o, _ = DC.run(q, k, v, g, be, bw, s0, per_channel=per_channel)
    B, T, H, dk = q.shape
    G = np.cumsum(g if per_channel else np.repeat(g[..., None], dk, -1), axis=1)   # log P_t
    for b in range(B):
        for h in range(H):
            for t in range(T):
                ref = s0[b, h].T @ (np.exp(G[b, t, h]) * q[b, t, h])
                for s in range(t + 1):
                    w = np.sum(q[b, t, h] * np.exp(G[b, t, h] - G[b, s, h]) * k[b, s, h])
                    ref = ref + bw[b, s, h] * w * v[b, s, h]
                np.testing.assert_allclose(o[b, t, h], ref, rtol=1e-11, atol=1e-12)


def test_no_write_is_the_coupled_rule_without_values():
    q, k, v, g, be, _, s0 = _case(True, 3)
    o1, s1 = DC.run(q, k, v, g, be, np.zeros_like(be), s0, per_channel=True)
    o2, s2 = oracle.run(q, k, np.zeros_like(v), g, be, s0, per_channel=True, threads=1)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-13)


def test_literal_transition_matrices():
    """S_t = (I - be k k^T) Diag(a) S_{t-1} + bw k v^T with explicit dk x dk
    matrices, one (b, h) at a time."""
    q, k, v, g, be, bw, s0 = _case(True, 4, B=1, H=1)
    o, sT = DC.run(q, k, v, g, be, bw, s0, per_channel=True)
    S = s0[0, 0].copy()
    dk = S.shape[0]
    for t in range(q.shape[1]):
        kk = k[0, t, 0]
        M = (np.eye(dk) - be[0, t, 0] * np.outer(kk, kk)) @ np.diag(np.exp(g[0, t, 0]))
        S = M @ S + bw[0, t, 0] * np.outer(kk, v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S.T @ q[0, t, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sT[0, 0], S, rtol=1e-12, atol=1e-13)
