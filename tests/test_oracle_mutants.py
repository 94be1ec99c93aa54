"""Planted mistakes: each plausible error in a recurrence implementation must be
rejected by at least one oracle pin (CPU only).

The mutants are small NumPy token loops written here, each with one mistake;
the oracle itself is not modified.  A mutant that passed every pin would mean
the pins cannot tell that mistake from the method.
"""
import numpy as np
import pytest

from tests import oracle_pins as pins


def _loop(q, k, v, g, beta, s0, *, per_channel, mistake):
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            for t in range(T):
                kt, vt, qt, bt = k[b, t, h], v[b, t, h], q[b, t, h], beta[b, t, h]
                a = np.exp(g[b, t, h]) if per_channel else np.full(dk, np.exp(g[b, t, h]))
                if mistake == "exp_of_minus_g":
                    a = 1.0 / a
                if mistake == "decay_columns":
                    Sp = S * a[None, :dv] if dk == dv else S * np.resize(a, dv)[None, :]
                else:
                    Sp = a[:, None] * S
                if mistake == "decay_after_erase":
                    e = vt - S.T @ kt
                    Snew = a[:, None] * (S + bt * np.outer(kt, e))
                elif mistake == "error_without_decay":
                    Snew = Sp + bt * np.outer(kt, vt - S.T @ kt)
                elif mistake == "error_sign":
                    Snew = Sp + bt * np.outer(kt, vt + Sp.T @ kt)
                elif mistake == "beta_only_on_write":
                    Snew = Sp - np.outer(kt, Sp.T @ kt) + bt * np.outer(kt, vt)
                elif mistake == "no_erase":
                    Snew = Sp + bt * np.outer(kt, vt)
                else:
                    Snew = Sp + bt * np.outer(kt, vt - Sp.T @ kt)
                if mistake == "output_from_previous_state":
                    o = S.T @ qt
                elif mistake == "output_transposed":
                    o = (Snew @ qt[:dv]) if dk == dv else Snew[:dv, :dv] @ qt[:dv]
                elif mistake == "key_for_query":
                    o = Snew.T @ kt
                else:
                    o = Snew.T @ qt
                out[b, t, h] = o
                S = Snew
            sT[b, h] = S
    return out, sT


MISTAKES = ["exp_of_minus_g", "decay_columns", "decay_after_erase", "error_without_decay",
            "error_sign", "beta_only_on_write", "no_erase", "output_from_previous_state",
            "output_transposed", "key_for_query"]


def test_unmutated_loop_passes_every_pin():
    impl = lambda *a, per_channel: _loop(*a, per_channel=per_channel, mistake=None)  # noqa: E731
    for pin in pins.ALL_PINS:
        pin(impl)


@pytest.mark.parametrize("mistake", MISTAKES)
def test_mutant_is_rejected(mistake):
    impl = lambda *a, per_channel: _loop(*a, per_channel=per_channel, mistake=mistake)  # noqa: E731
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the mistake {mistake!r}"
