"""Pins of ``oracle.rel_err``, the tolerance rule every parity test uses.

The rule (the workloads state each tolerance as max|got - ref| <= tol * rms(o)):
the largest absolute difference over ALL elements, divided by the root mean
square of the REFERENCE over all elements.  Each case below is computed by
hand and is chosen so that a plausible slip gives a different number:
rms taken of ``got`` instead of ``ref``, a per-row (axis-wise) normalisation,
the mean of |difference| in place of its maximum, or a NaN that slips through.
"""
import math

import numpy as np
import torch

import oracle


def test_hand_computed_vector():
    # max|d| = 1; rms(ref) = sqrt((9 + 16) / 2) = sqrt(12.5).
    # rms(got) = sqrt(17) and mean|d| = 0.5 would give other values.
    got = oracle.rel_err(np.array([3.0, 5.0]), np.array([3.0, 4.0]))
    assert math.isclose(got, 1.0 / math.sqrt(12.5), rel_tol=1e-15)
    assert not math.isclose(got, 1.0 / math.sqrt(17.0), rel_tol=1e-6)


def test_normalisation_is_over_the_whole_tensor():
    # rms over all four elements = sqrt((1 + 1 + 100 + 100) / 4) = sqrt(50.5);
    # a row-wise rule would give 1 / 1 = 1 for the first row.
    ref = np.array([[1.0, 1.0], [10.0, 10.0]])
    got = np.array([[2.0, 1.0], [10.0, 10.0]])
    assert math.isclose(oracle.rel_err(got, ref), 1.0 / math.sqrt(50.5), rel_tol=1e-15)


def test_maximum_not_mean_of_the_differences():
    # Differences 0, 0, 0, 4: max 4, mean 1.  rms(ref) = sqrt(4) = 2.
    ref = np.full(4, 2.0)
    got = np.array([2.0, 2.0, 2.0, -2.0])
    assert math.isclose(oracle.rel_err(got, ref), 2.0, rel_tol=1e-15)


def test_sign_of_the_difference_does_not_matter():
    ref = np.array([1.0, -1.0, 1.0, -1.0])            # rms 1
    assert oracle.rel_err(ref + np.array([0, 0, 0, -0.25]), ref) == 0.25
    assert oracle.rel_err(ref + np.array([0, 0.25, 0, 0]), ref) == 0.25


def test_zero_reference_falls_back_to_the_absolute_difference():
    assert oracle.rel_err(np.array([0.0, 0.5]), np.zeros(2)) == 0.5
    assert oracle.rel_err(np.zeros(3), np.zeros(3)) == 0.0


def test_a_nan_never_passes():
    r = oracle.rel_err(np.array([1.0, float("nan")]), np.array([1.0, 1.0]))
    assert not (r <= 1e30)


def test_torch_inputs_are_read_exactly():
    # bf16 holds 3 and 5 exactly; the rule sees the same numbers as above.
    got = torch.tensor([3.0, 5.0], dtype=torch.bfloat16)
    ref = torch.tensor([3.0, 4.0], dtype=torch.float32)
    assert math.isclose(oracle.rel_err(got, ref), 1.0 / math.sqrt(12.5), rel_tol=1e-15)


# ---- the pins reject plausible slips ----------------------------------------
def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _rms_of_got(got, ref):
    got, ref = _f64(got), _f64(ref)
    return float(np.max(np.abs(got - ref)) / np.sqrt(np.mean(got * got)))


def _row_wise(got, ref):
    got, ref = np.atleast_2d(_f64(got)), np.atleast_2d(_f64(ref))
    rms = np.sqrt(np.mean(ref * ref, axis=-1))
    return float(np.max(np.max(np.abs(got - ref), axis=-1) / rms))


def _mean_abs(got, ref):
    got, ref = _f64(got), _f64(ref)
    return float(np.mean(np.abs(got - ref)) / np.sqrt(np.mean(ref * ref)))


def _nan_blind(got, ref):
    got, ref = _f64(got), _f64(ref)
    return float(np.nanmax(np.abs(got - ref)) / np.sqrt(np.mean(ref * ref)))


def _cases():
    yield np.array([3.0, 5.0]), np.array([3.0, 4.0]), 1.0 / math.sqrt(12.5)
    yield np.array([[2.0, 1.0], [10.0, 10.0]]), np.array([[1.0, 1.0], [10.0, 10.0]]), 1.0 / math.sqrt(50.5)
    yield np.array([2.0, 2.0, 2.0, -2.0]), np.full(4, 2.0), 2.0
    yield np.array([1.0, float("nan")]), np.array([1.0, 1.0]), float("nan")


def _passes(f):
    for got, ref, want in _cases():
        r = f(got, ref)
        if math.isnan(want):
            if not math.isnan(r):
                return False
        elif not math.isclose(r, want, rel_tol=1e-12):
            return False
    return True


def test_pins_accept_the_rule_and_reject_its_slips():
    assert _passes(oracle.rel_err)
    for mutant in (_rms_of_got, _row_wise, _mean_abs, _nan_blind):
        assert not _passes(mutant), mutant.__name__
