"""The soft-capping polynomial of the forward kernel (kTanhPoly in
fwd_common.cuh): tanh(t) = t * P(t^2) on |t| <= kTanhPolyRange.  Its
coefficients, read from the kernel source, are evaluated here as the kernel
evaluates them (float32 Horner in t^2) and checked against tanh in fp64: the
relative error stays below 2e-7 over the whole range, and the leading terms
agree with the series tanh(t) = t - t^3/3 + 2 t^5/15 - ... to the accuracy of
a least-maximum-error fit."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "exact_attention_157_b200", "csrc", "fwd_common.cuh")


def constants():
    text = open(SRC).read()
    terms = int(re.search(r"constexpr int kTanhPolyTerms = (\d+);", text).group(1))
    rng = float(re.search(r"constexpr float kTanhPolyRange = ([0-9.eE+-]+)f;", text).group(1))
    body = re.search(r"constexpr float kTanhPoly\[kTanhPolyTerms\] = \{([^}]*)\}", text).group(1)
    coef = [np.float32(float(x.strip().rstrip("f"))) for x in body.split(",")]
    assert len(coef) == terms
    return rng, coef


def horner_f32(t, coef):
    t = t.astype(np.float32)
    w = (t * t).astype(np.float32)
    h = np.full_like(w, coef[-1])
    for c in coef[-2::-1]:
        h = (h * w + c).astype(np.float32)
    return (t * h).astype(np.float32)


def test_relative_error_over_the_range():
    rng, coef = constants()
    t = np.linspace(-rng, rng, 400001, dtype=np.float32)
    t = t[t != 0]
    got = horner_f32(t, coef).astype(np.float64)
    ref = np.tanh(t.astype(np.float64))
    assert np.max(np.abs(got - ref) / np.abs(ref)) < 2e-7


def test_tiny_arguments_and_oddness():
    rng, coef = constants()
    t = np.array([1e-30, 1e-10, 1e-4, 0.0], dtype=np.float32)
    got = horner_f32(t, coef)
    np.testing.assert_array_equal(got[:3], t[:3])  # tanh(t) = t to float precision
    assert got[3] == 0.0
    s = np.linspace(0.01, rng, 1001, dtype=np.float32)
    np.testing.assert_array_equal(horner_f32(-s, coef), -horner_f32(s, coef))


def test_leading_terms_follow_the_series():
    _, coef = constants()
    assert coef[0] == np.float32(1.0)
    assert abs(coef[1] + 1.0 / 3.0) < 1e-5
    assert abs(coef[2] - 2.0 / 15.0) < 1e-3
    assert abs(coef[3] + 17.0 / 315.0) < 2e-3


def test_a_planted_slip_fails():
    rng, coef = constants()
    t = np.linspace(-rng, rng, 20001, dtype=np.float32)
    t = t[t != 0]
    ref = np.tanh(t.astype(np.float64))
    for i in range(1, len(coef)):
        bad = list(coef)
        bad[i] = np.float32(bad[i] * 1.01)
        got = horner_f32(t, bad).astype(np.float64)
        assert np.max(np.abs(got - ref) / np.abs(ref)) > 2e-7, f"1 % slip of term {i} not seen"
