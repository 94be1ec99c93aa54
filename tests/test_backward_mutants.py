"""The finite-difference pin of the gradient oracle rejects plausible slips.

A separate NumPy copy of the reverse sweep (one (b, h), plain loops) takes a
``mutant`` switch that plants one mistake; the unmutated copy must agree with
central differences of the C forward oracle, and every mutant must not.
"""
import numpy as np
import pytest

import oracle

MUTANTS = [None, "drop_q_do", "sign_erase", "beta_on_dv_missing", "decay_after", "dk_write_term",
           "dbeta_uses_u", "dg_without_a"]


def _reverse(q, k, v, g, beta, s0, do, dsT, mutant):
    T, dk = q.shape
    S = [s0.copy()]
    for t in range(T):
        a = np.exp(g[t])
        Sp = a[:, None] * S[-1]
        e = v[t] - Sp.T @ k[t]
        S.append(Sp + beta[t] * np.outer(k[t], e))
    dS = dsT.copy()
    grads = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta))}
    for t in range(T - 1, -1, -1):
        a = np.exp(g[t])
        Sp = a[:, None] * S[t]
        e = v[t] - Sp.T @ k[t]
        if mutant != "drop_q_do":
            dS = dS + np.outer(q[t], do[t])
        grads["q"][t] = S[t + 1] @ do[t]
        du = dS.T @ k[t]
        grads["k"][t] = dS @ (beta[t] * e) if mutant != "dk_write_term" else 0.0
        de = beta[t] * du if mutant != "beta_on_dv_missing" else du
        grads["beta"][t] = du @ (e if mutant != "dbeta_uses_u" else beta[t] * e)
        grads["v"][t] = de
        dSp = dS - np.outer(k[t], de) if mutant != "sign_erase" else dS + np.outer(k[t], de)
        grads["k"][t] = grads["k"][t] - Sp @ de
        da = np.sum(dSp * S[t], axis=1)
        grads["g"][t] = da * a if mutant != "dg_without_a" else da
        dS = a[:, None] * dSp if mutant != "decay_after" else dSp
    return grads


def _fd(x, do, dsT, name):
    h = 1e-6
    fd = np.zeros_like(x[name])
    for idx in np.ndindex(x[name].shape):
        vals = []
        for sgn in (1, -1):
            y = {n: a.copy() for n, a in x.items()}
            y[name][idx] += sgn * h
            o, sT = oracle.run(*(y[n][None, :, None] for n in ("q", "k", "v", "g", "beta")),
                               y["s0"][None, None], per_channel=True, threads=1)
            vals.append(np.sum(do * o[0, :, 0]) + np.sum(dsT * sT[0, 0]))
        fd[idx] = (vals[0] - vals[1]) / (2 * h)
    return fd


@pytest.fixture(scope="module")
def case():
    rng = np.random.default_rng(11)
    T, dk, dv = 4, 3, 2
    x = dict(q=rng.normal(size=(T, dk)), k=rng.normal(size=(T, dk)) / np.sqrt(dk),
             v=rng.normal(size=(T, dv)), g=-np.abs(rng.normal(size=(T, dk))) * 0.5,
             beta=rng.uniform(0.2, 0.9, size=T), s0=rng.normal(size=(dk, dv)) * 0.3)
    do, dsT = rng.normal(size=(T, dv)), rng.normal(size=(dk, dv))
    fds = {n: _fd(x, do, dsT, n) for n in ("q", "k", "v", "g", "beta")}
    return x, do, dsT, fds


@pytest.mark.parametrize("mutant", MUTANTS)
def test_finite_differences_reject_every_mutant(case, mutant):
    x, do, dsT, fds = case
    got = _reverse(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], do, dsT, mutant)
    worst = max(float(np.max(np.abs(got[n] - fds[n]))) for n in fds)
    if mutant is None:
        assert worst <= 1e-7
    else:
        assert worst > 1e-3, mutant
