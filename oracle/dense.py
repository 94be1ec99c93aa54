"""Tiny-size fp64 NumPy forms of the recurrence -- TEST INFRASTRUCTURE ONLY.

Two forms that reach the token recurrence by different algebra, used to pin
the C oracle (``oracle.run``) on small inputs:

``transition_form``
    The formula exactly as printed in the Atomic-GDN2 model card, section 2.1:
    an explicit dk x dk transition matrix per token,
        A_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
        S_t = A_t S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.

``chunk_form``
    The chunkwise-parallel mode ("Gated DeltaNet" entity trail, finding of
    2026-07-29: the chunkwise mode computes the same mathematics as the
    recurrent one).  Inside a chunk of C tokens with initial state S0 and
    cumulative log-decay Gamma_r = sum_{s<=r} g_s (scalar or per key channel):
        A_rj = beta_r k_r^T Diag(exp(Gamma_r - Gamma_j)) k_j     (j < r)
        (I + A) U = Diag(beta) V - Diag(beta) (K * exp(Gamma)) S0
        P_rj = q_r^T Diag(exp(Gamma_r - Gamma_j)) k_j            (j <= r)
        O    = (Q * exp(Gamma)) S0 + P U
        S_C  = Diag(exp(Gamma_last)) S0 + (K * exp(Gamma_last - Gamma))^T U
    The triangular system is solved with ``numpy.linalg.solve`` (no explicit
    inverse, no blocking).  Derivation: unroll the recurrence over the chunk;
    u_r = beta_r (v_r - S'_r^T k_r) is the corrected value written at token r.
"""
from __future__ import annotations

import numpy as np


def _alpha_vec(g_t, dk, per_channel):
    return np.exp(g_t) if per_channel else np.full(dk, np.exp(g_t))


def transition_form(q, k, v, g, beta, s0=None, *, per_channel: bool):
    """Literal transition-matrix product. Shapes as ``oracle.run``; fp64."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    eye = np.eye(dk)
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            for t in range(T):
                kt = k[b, t, h]
                a = _alpha_vec(g[b, t, h], dk, per_channel)
                A = (eye - beta[b, t, h] * np.outer(kt, kt)) @ np.diag(a)
                S = A @ S + beta[b, t, h] * np.outer(kt, v[b, t, h])
                out[b, t, h] = S.T @ q[b, t, h]
            sT[b, h] = S
    return out, sT


def chunk_form(q, k, v, g, beta, s0=None, *, per_channel: bool, chunk: int):
    """Chunkwise closed form (see module docstring). Shapes as ``oracle.run``."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            for t0 in range(0, T, chunk):
                t1 = min(T, t0 + chunk)
                n = t1 - t0
                Q = q[b, t0:t1, h]
                K = k[b, t0:t1, h]
                V = v[b, t0:t1, h]
                bt = beta[b, t0:t1, h]
                if per_channel:
                    G = np.cumsum(g[b, t0:t1, h], axis=0)            # [n, dk]
                else:
                    G = np.repeat(np.cumsum(g[b, t0:t1, h])[:, None], dk, axis=1)
                A = np.zeros((n, n))
                P = np.zeros((n, n))
                for r in range(n):
                    for j in range(r + 1):
                        d = np.exp(G[r] - G[j])
                        P[r, j] = np.dot(Q[r] * d, K[j])
                        if j < r:
                            A[r, j] = bt[r] * np.dot(K[r] * d, K[j])
                E = np.exp(G)
                rhs = bt[:, None] * V - (bt[:, None] * K * E) @ S
                U = np.linalg.solve(np.eye(n) + A, rhs)
                out[b, t0:t1, h] = (Q * E) @ S + P @ U
                S = np.diag(np.exp(G[-1])) @ S + (K * np.exp(G[-1][None, :] - G)).T @ U
            sT[b, h] = S
    return out, sT
