"""The segment-parallel prefill's mathematics, pinned on the fp64 oracle (CPU).

The segment path cuts a sequence into segments that run from a zero state
and corrects them afterwards.  Two facts carry it:

* the state map of a stretch of tokens is affine in its start state (it
  follows from the recurrence of the Atomic-GDN2 model card, section 2.1):
  S_t = M_t S_start + S_t(0) and o_t = o_t(0) + S_start^T (M_t^T q_t), where
  M_t is the product of the per-token maps (I - beta k k^T) Diag(alpha) and
  S_t(0), o_t(0) the zero-start run.  M_t itself is the state of a run with
  v = 0 from the identity, and M_t^T q_t its output.
* on the contracting domain (g <= 0 in every channel, 0 <= beta |k|^2 <= 2)
  every per-token map has spectral norm <= 1, so a transition whose entries
  have all fallen to eps stays below |M|_2 <= |M|_F <= dk eps for the rest of
  the segment: dropping it changes an output by at most dk eps |S_start| |q|.
  Outside the domain (beta |k|^2 > 2) the map can grow, which is why the
  kernel checks the domain before it ends a transition.

Every quantity below comes from oracle.run on small inputs.
"""
import numpy as np
import pytest

import oracle

D = 16


def _inputs(T, gate, seed, beta_scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, 1, D))
    k = rng.standard_normal((1, T, 1, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, D))
    beta = beta_scale / (1.0 + np.exp(-rng.standard_normal((1, T, 1))))
    shape = (1, T, 1, D) if gate == "channel" else (1, T, 1)
    g = -np.minimum(np.log1p(np.exp(rng.standard_normal(shape))), 5.0) * 0.3
    return q, k, v, g, beta


def _transition(q, k, g, beta, per_channel):
    """M_t^T q_t per token and the segment's M (a run with v = 0 from I)."""
    zeros = np.zeros_like(k)
    eye = np.eye(D)[None, None]
    return oracle.run(q, k, zeros, g, beta, eye, per_channel=per_channel)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_segment_state_map_is_affine(gate):
    T, cut = 120, 50
    q, k, v, g, beta = _inputs(T, gate, seed=1)
    s0 = np.random.default_rng(2).standard_normal((1, 1, D, D)) * 0.3
    pc = gate == "channel"
    o_full, s_full = oracle.run(q, k, v, g, beta, s0, per_channel=pc)
    sl = lambda x: x[:, cut:]
    _, s_mid = oracle.run(q[:, :cut], k[:, :cut], v[:, :cut], g[:, :cut], beta[:, :cut], s0,
                          per_channel=pc)
    o_zero, s_zero = oracle.run(sl(q), sl(k), sl(v), sl(g), sl(beta), None, per_channel=pc)
    w, m = _transition(sl(q), sl(k), sl(g), sl(beta), pc)
    # S_end = M S_mid + S_end(0); o_t = o_t(0) + S_mid^T (M_t^T q_t)
    np.testing.assert_allclose(s_full[0, 0], m[0, 0] @ s_mid[0, 0] + s_zero[0, 0], atol=1e-12)
    corr = np.einsum("ij,ti->tj", s_mid[0, 0], w[0, :, 0])
    np.testing.assert_allclose(o_full[0, cut:, 0], o_zero[0, :, 0] + corr, atol=1e-12)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_transitions_contract_on_the_domain(gate):
    """Every prefix M_t of a transition has |M_t|_2 <= 1, and once its entries
    are below eps the later prefixes stay below dk eps in spectral norm."""
    T = 80
    q, k, v, g, beta = _inputs(T, gate, seed=3)
    pc = gate == "channel"
    norms, maxabs = [], []
    for t in range(1, T + 1):
        _, m = _transition(q[:, :t], k[:, :t], g[:, :t], beta[:, :t], pc)
        norms.append(np.linalg.norm(m[0, 0], 2))
        maxabs.append(np.abs(m[0, 0]).max())
    assert max(norms) <= 1.0 + 1e-12
    assert all(b <= a + 1e-15 for a, b in zip(norms, norms[1:]))     # non-increasing
    for i, eps in enumerate(maxabs):
        assert max(norms[i:]) <= D * eps + 1e-15


def test_a_map_outside_the_domain_can_grow():
    """beta |k|^2 > 2 breaks the contraction: (I - beta k k^T) has the
    eigenvalue 1 - beta |k|^2 < -1 along k, so a transition can grow and the
    kernel must not end it early (it checks beta (K K^T)_rr <= 2)."""
    q, k, v, g, beta = _inputs(1, "scalar", seed=4)
    g[:] = 0.0
    beta[:] = 2.5
    _, m = _transition(q, k, g, beta, False)
    assert np.linalg.norm(m[0, 0], 2) == pytest.approx(1.5, rel=1e-12)
