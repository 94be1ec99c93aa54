"""Pins for the fp64 oracle: facts fixed by the method's formula and by
mathematics, each checked against an implementation passed in as ``impl``.

``impl(q, k, v, g, beta, s0, per_channel=...) -> (out, s_final)`` has the
signature of ``oracle.run``.  The real oracle must pass every pin; each
planted mistake in ``tests/test_oracle_mutants.py`` must fail at least one.

Formula: Atomic-GDN2 model card, section 2.1 "Gated DeltaNet-2".
Invariants I1-I10 are derived from it (β=0/α=1 freezes the state, an exact
β=1 write with a unit key overwrites, per-channel gates equal across channels
reduce to the scalar gate, ...).
"""
from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).resolve().parent / "golden"


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_case(seed, B=2, T=9, H=2, dk=5, dv=3, per_channel=True, s0=True, beta_one=False):
    r = _rng(seed)
    q = _unit_rows(r.standard_normal((B, T, H, dk)))
    k = _unit_rows(r.standard_normal((B, T, H, dk)))
    v = r.standard_normal((B, T, H, dv))
    beta = np.ones((B, T, H)) if beta_one else 1.0 / (1.0 + np.exp(-r.standard_normal((B, T, H))))
    gshape = (B, T, H, dk) if per_channel else (B, T, H)
    g = -np.minimum(np.log1p(np.exp(r.standard_normal(gshape))), 5.0)
    S0 = r.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, g, beta, S0


def close(a, b, tol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b)))) if b.size else 1.0
    assert err <= tol * scale, f"{what}: max err {err:.3e} > {tol:.1e}*{scale:.3g}"


# --- I1: beta = 0 and g = 0 freeze the state ------------------------------------------
def pin_frozen_state(impl):
    for pc in (False, True):
        q, k, v, g, beta, S0 = random_case(11, per_channel=pc)
        g = np.zeros_like(g)
        beta = np.zeros_like(beta)
        out, sT = impl(q, k, v, g, beta, S0, per_channel=pc)
        close(sT, S0, what="I1 final state")
        close(out, np.einsum("bhij,bthi->bthj", S0, q), what="I1 o_t = S0^T q_t")


# --- I2: an exact write with beta = 1 and a unit key is read back exactly --------------
def pin_exact_overwrite(impl):
    # Orthonormal keys, alpha = 1, S0 = 0: write (k_i, v_i), then read with q = k_i.
    dk, dv, m = 6, 4, 4
    r = _rng(21)
    basis, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    keys = basis[:, :m].T                                    # m orthonormal rows
    vals = r.standard_normal((m, dv))
    T = 2 * m
    q = np.zeros((1, T, 1, dk)); k = np.zeros((1, T, 1, dk)); v = np.zeros((1, T, 1, dv))
    beta = np.zeros((1, T, 1))
    for i in range(m):
        k[0, i, 0] = keys[i]; v[0, i, 0] = vals[i]; beta[0, i, 0] = 1.0
        q[0, i, 0] = keys[0]                                 # reads key 0 while writing
        q[0, m + i, 0] = keys[i]                             # read phase: beta = 0
        k[0, m + i, 0] = keys[(i + 1) % m]
        v[0, m + i, 0] = r.standard_normal(dv)
    for pc in (False, True):
        g = np.zeros((1, T, 1, dk)) if pc else np.zeros((1, T, 1))
        out, _ = impl(q, k, v, g, beta, None, per_channel=pc)
        for i in range(m):
            close(out[0, m + i, 0], vals[i], what=f"I2 read-back of value {i}")
            close(out[0, i, 0], vals[0], what=f"I2 key 0 while writing {i}")
    # Stronger form: any decay, any prior state, beta = 1, unit key => S_t^T k_t = v_t.
    for pc in (False, True):
        q, k, v, g, beta, S0 = random_case(22, per_channel=pc, beta_one=True)
        out, _ = impl(k.copy(), k, v, g, beta, S0, per_channel=pc)
        close(out, v, tol=1e-11, what="I2 S_t^T k_t = v_t after a beta=1 write")


# --- I3: per-channel gate equal across channels == scalar gate ------------------------
def pin_channel_broadcast(impl):
    q, k, v, g, beta, S0 = random_case(31, per_channel=False)
    dk = q.shape[-1]
    o_s, s_s = impl(q, k, v, g, beta, S0, per_channel=False)
    g_c = np.repeat(g[..., None], dk, axis=-1)
    o_c, s_c = impl(q, k, v, g_c, beta, S0, per_channel=True)
    close(o_c, o_s, tol=1e-13, what="I3 outputs")
    close(s_c, s_s, tol=1e-13, what="I3 states")


# --- I4: literal transition matrices and the chunk closed form -----------------------
def pin_dense_forms(impl):
    from oracle import dense
    for pc in (False, True):
        q, k, v, g, beta, S0 = random_case(41, per_channel=pc)
        out, sT = impl(q, k, v, g, beta, S0, per_channel=pc)
        o_t, s_t = dense.transition_form(q, k, v, g, beta, S0, per_channel=pc)
        close(out, o_t, what="I4 transition form, outputs")
        close(sT, s_t, what="I4 transition form, state")
        for C in (1, 2, 4, 9):
            o_c, s_c = dense.chunk_form(q, k, v, g, beta, S0, per_channel=pc, chunk=C)
            close(out, o_c, tol=1e-11, what=f"I4 chunk form C={C}, outputs")
            close(sT, s_c, tol=1e-11, what=f"I4 chunk form C={C}, state")


# --- I5: beta = 0 => pure cumulative decay of the rows of S0 -------------------------
def pin_pure_decay(impl):
    for pc in (False, True):
        q, k, v, g, beta, S0 = random_case(51, per_channel=pc)
        beta = np.zeros_like(beta)
        out, sT = impl(q, k, v, g, beta, S0, per_channel=pc)
        G = np.cumsum(g, axis=1)                              # [B,T,H(,dk)]
        if not pc:
            G = np.repeat(G[..., None], q.shape[-1], axis=-1)
        St = np.exp(G)[..., None] * S0[:, None]               # [B,T,H,dk,dv]: rows scaled
        close(out, np.einsum("bthij,bthi->bthj", St, q), what="I5 outputs")
        close(sT, St[:, -1], what="I5 final state")


# --- I6: the map (S0, V) -> (o, S_T) is linear for fixed q, k, g, beta ----------------
def pin_linearity(impl):
    q, k, v, g, beta, S0 = random_case(61, per_channel=True)
    o_a, s_a = impl(q, k, v, g, beta, S0, per_channel=True)
    o_b, s_b = impl(q, k, np.zeros_like(v), g, beta, S0, per_channel=True)
    o_c, s_c = impl(q, k, v, g, beta, np.zeros_like(S0), per_channel=True)
    close(o_a, o_b + o_c, tol=1e-12, what="I6 outputs")
    close(s_a, s_b + s_c, tol=1e-12, what="I6 states")


# --- I7: T = 1, dk = dv = 1 closed form -------------------------------------------------
def pin_scalar_closed_form(impl):
    for (s0, g, b, kk, vv, qq) in [(0.5, -0.3, 0.25, 0.6, 2.0, -1.5), (-1.0, 0.0, 1.0, 1.0, 0.5, 2.0),
                                   (2.0, -5.0, 0.9, -0.7, -1.0, 0.3)]:
        a = math.exp(g)
        s1 = a * s0 + b * kk * (vv - a * s0 * kk)            # delta form with one channel
        o1 = s1 * qq
        arr = lambda x: np.array(x, dtype=np.float64).reshape(1, 1, 1, 1)  # noqa: E731
        out, sT = impl(arr(qq), arr(kk), arr(vv), np.array([[[g]]]), np.array([[[b]]]),
                       arr(s0), per_channel=False)
        close(out.reshape(()), o1, what="I7 output")
        close(sT.reshape(()), s1, what="I7 state")


def pin_hand_worked(impl):
    data = json.loads((GOLDEN / "hand_worked.json").read_text())
    for case in data["cases"]:
        conv = lambda x: np.vectorize(lambda e: math.log(0.5) if e == "ln0.5" else float(e),  # noqa: E731
                                      otypes=[np.float64])(np.array(x, dtype=object))
        q, k, v, g, beta = (np.swapaxes(conv(case[n]), 0, 1) for n in ("q", "k", "v", "g", "beta"))
        s0 = conv(case["s0"])
        out, sT = impl(q, k, v, g, beta, s0, per_channel=case["per_channel"])
        close(np.swapaxes(out, 0, 1), conv(case["out"]), tol=1e-12, what=case["name"] + " outputs")
        close(sT, conv(case["s_final"]), tol=1e-12, what=case["name"] + " state")


# --- I8: norm bound with unit keys, beta in [0, 1], g <= 0 ----------------------------
def pin_norm_bound(impl):
    q, k, v, g, beta, S0 = random_case(81, B=1, T=12, H=1, per_channel=True)
    S = S0
    for t in range(q.shape[1]):
        sl = slice(t, t + 1)
        _, S_next = impl(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], S, per_channel=True)
        bound = np.linalg.norm(S) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert np.linalg.norm(S_next) <= bound * (1 + 1e-12), "I8 norm bound violated"
        S = S_next


# --- I9: splitting the sequence and carrying the state changes nothing --------------
def pin_split_sequence(impl):
    q, k, v, g, beta, S0 = random_case(91, T=11, per_channel=True)
    out, sT = impl(q, k, v, g, beta, S0, per_channel=True)
    for T1 in (0, 1, 5, 10, 11):
        a = slice(0, T1)
        b = slice(T1, None)
        o1, s1 = impl(q[:, a], k[:, a], v[:, a], g[:, a], beta[:, a], S0, per_channel=True)
        o2, s2 = impl(q[:, b], k[:, b], v[:, b], g[:, b], beta[:, b], s1, per_channel=True)
        close(np.concatenate([o1, o2], axis=1), out, what=f"I9 split at {T1}, outputs")
        close(s2, sT, what=f"I9 split at {T1}, state")


# --- I10: prefill over T tokens == T single-token steps -------------------------------
def pin_prefill_equals_steps(impl):
    q, k, v, g, beta, S0 = random_case(101, T=6, per_channel=True)
    out, sT = impl(q, k, v, g, beta, S0, per_channel=True)
    S = S0
    for t in range(q.shape[1]):
        sl = slice(t, t + 1)
        o_t, S = impl(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], S, per_channel=True)
        close(o_t[:, 0], out[:, t], what=f"I10 step {t}")
    close(S, sT, what="I10 final state")


ALL_PINS = [pin_frozen_state, pin_exact_overwrite, pin_channel_broadcast, pin_dense_forms,
            pin_pure_decay, pin_linearity, pin_scalar_closed_form, pin_hand_worked,
            pin_norm_bound, pin_split_sequence, pin_prefill_equals_steps]
