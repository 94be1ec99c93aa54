"""fp64 oracle of the decoupled erase / write form of the recurrence -- TEST
INFRASTRUCTURE ONLY (same import rule as the rest of ``oracle/``).

PARITY UNPINNED as to the form itself: the "Gated DeltaNet" entity trail
(finding of 2026-05-22) describes Gated DeltaNet-2 as decoupling the erase
and the write of the delta rule with separate gates instead of one scalar,
and gives no formula.  The reading taken here is the plainest one, with the
model card's recurrence (section 2.1) as its special case: the scalar beta
of the erase term and the scalar beta of the write term become two gates,
one value each per (token, head):

    S'_t = Diag(a_t) S_{t-1},  a_t = exp(g_t)           (decay first)
    S_t  = S'_t - be_t k_t (k_t^T S'_t) + bw_t k_t v_t^T
         = (I - be_t k_t k_t^T) S'_t + bw_t k_t v_t^T
    o_t  = S_t^T q_t

The arithmetic of this reading is pinned (tests/test_decoupled_oracle.py):
be = bw reproduces the coupled C oracle, be = 0 is gated linear attention
with its explicit sum, bw = 0 is the coupled rule with v = 0, and the
literal dk x dk transition matrices give the same states.
Layouts as the library's: [B, T, H, ...]; states [B, H, dk, dv].
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype.is_floating_point:
            x = x.double()
        return x.numpy()
    return np.asarray(x, dtype=np.float64)


def run(q, k, v, g, beta_erase, beta_write, s0=None, *, per_channel: bool):
    """Returns (o [B, T, H, dv], S_T [B, H, dk, dv]) in fp64."""
    q, k, v, g, be, bw, s0 = (_f64(x) for x in (q, k, v, g, beta_erase, beta_write, s0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if s0 is None else s0.copy()
    o = np.zeros((B, T, H, dv))
    for t in range(T):
        a = np.exp(g[:, t]) if per_channel else np.exp(g[:, t])[..., None]
        Sp = a[..., None] * S
        x = np.einsum("bhij,bhi->bhj", Sp, k[:, t])          # k^T S'
        u = bw[:, t][..., None] * v[:, t] - be[:, t][..., None] * x
        S = Sp + k[:, t][..., :, None] * u[..., None, :]
        o[:, t] = np.einsum("bhij,bhi->bhj", S, q[:, t])
    return o, S
