"""fp64 oracle of the gradients of the Gated DeltaNet recurrence -- TEST
INFRASTRUCTURE ONLY (same import rule as the rest of ``oracle/``).

The forward is the recurrence of the Atomic-GDN2 model card, section 2.1
("Gated DeltaNet-2"), in its delta-rule form, token by token:

    a_t  = exp(g_t)                         scalar, or one value per key channel
    S'_t = Diag(a_t) S_{t-1}                decay first
    e_t  = v_t - S'_t^T k_t                 the error the delta rule writes
    S_t  = S'_t + beta_t k_t e_t^T          = (I - beta k k^T) S'_t + beta k v^T
    o_t  = S_t^T q_t

Its reverse-mode derivative, taken step by step from the last token back to
the first (plain chain rule on the five lines above, in reverse order), with
dS the gradient of the loss with respect to S_t (the caller's dS_T, or 0):

    dS   += q_t do_t^T ;  dq_t = S_t do_t                       (o_t)
    du    = dS^T k_t   ;  dk_t = dS (beta_t e_t)                 (S_t, u = beta e)
    de    = beta_t du  ;  dbeta_t = du . e_t ;  dv_t = de        (u, e)
    dS'   = dS - k_t de^T ;  dk_t -= S'_t de                     (e)
    da_t  = sum over value columns of dS' * S_{t-1}  (summed over key channels
            too for a scalar gate) ;  dg_t = da_t a_t            (S', a = exp g)
    dS    = Diag(a_t) dS'

and dS_0 is the gradient of the initial state.  Every forward state is kept
(no recomputation), so memory grows as T * dk * dv per (b, h): small cases
only.  Layouts as the library's: [B, T, H, ...] token-major, states
[B, H, dk, dv].
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


def forward(q, k, v, g, beta, s0=None, *, per_channel: bool):
    """The recurrence; returns (o [B,T,H,dv], S_T [B,H,dk,dv], states) where
    states[t] = S_t for t = 0..T (fp64)."""
    q, k, v, g, beta, s0 = (_f64(x) for x in (q, k, v, g, beta, s0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if s0 is None else s0.copy()
    states = [S.copy()]
    o = np.zeros((B, T, H, dv))
    for t in range(T):
        a = np.exp(g[:, t]) if per_channel else np.exp(g[:, t])[..., None]   # [B,H,dk] or [B,H,1]
        Sp = a[..., None] * S
        e = v[:, t] - np.einsum("bhij,bhi->bhj", Sp, k[:, t])
        S = Sp + beta[:, t][..., None, None] * k[:, t][..., :, None] * e[..., None, :]
        o[:, t] = np.einsum("bhij,bhi->bhj", S, q[:, t])
        states.append(S.copy())
    return o, S, states


def backward(q, k, v, g, beta, s0, d_out, d_state=None, *, per_channel: bool):
    """Gradients of sum(d_out * o) + sum(d_state * S_T) with respect to every
    input.  Returns dict dq, dk, dv, dg, dbeta, ds0 (fp64; dg has g's shape)."""
    q, k, v, g, beta, s0, d_out, d_state = (_f64(x) for x in
                                            (q, k, v, g, beta, s0, d_out, d_state))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _, _, states = forward(q, k, v, g, beta, s0, per_channel=per_channel)
    dS = np.zeros((B, H, dk, dv)) if d_state is None else d_state.copy()
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dg = np.zeros_like(g)
    dbeta = np.zeros_like(beta)
    for t in range(T - 1, -1, -1):
        S_prev, S_t = states[t], states[t + 1]
        a = np.exp(g[:, t]) if per_channel else np.exp(g[:, t])[..., None]
        Sp = a[..., None] * S_prev
        e = v[:, t] - np.einsum("bhij,bhi->bhj", Sp, k[:, t])
        bt = beta[:, t][..., None]                                   # [B,H,1]
        # o_t = S_t^T q_t
        dS = dS + q[:, t][..., :, None] * d_out[:, t][..., None, :]
        dq[:, t] = np.einsum("bhij,bhj->bhi", S_t, d_out[:, t])
        # S_t = S'_t + k_t u_t^T with u_t = beta_t e_t
        du = np.einsum("bhij,bhi->bhj", dS, k[:, t])
        dkk[:, t] = np.einsum("bhij,bhj->bhi", dS, bt * e)
        de = bt * du
        dbeta[:, t] = np.sum(du * e, axis=-1)
        dvv[:, t] = de
        # e_t = v_t - S'_t^T k_t
        dSp = dS - k[:, t][..., :, None] * de[..., None, :]
        dkk[:, t] -= np.einsum("bhij,bhj->bhi", Sp, de)
        # S'_t = Diag(a_t) S_{t-1}, a_t = exp(g_t)
        da = np.sum(dSp * S_prev, axis=-1)                           # [B,H,dk]
        if per_channel:
            dg[:, t] = da * a
        else:
            dg[:, t] = np.sum(da, axis=-1) * a[..., 0]
        dS = a[..., None] * dSp
    return dict(dq=dq, dk=dkk, dv=dvv, dg=dg, dbeta=dbeta, ds0=dS)
