"""Pins of the calibration oracle: brute-force loops over (t, j <= t), the
total weight (each row weighs 1), closed forms on constructed logits,
monotonicity in the target, and the histogram solver within one bin of the
exact solver.  A mistake such as weighting by 1/t instead of 1/(t + 1), a
non-causal pair set, a reversed search direction or an off-by-one bin fails
one of them."""
import math

import numpy as np

from oracle import eta_calib_oracle as co


def test_brute_force_pairs_and_weights():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((6, 4))
    k = rng.standard_normal((6, 4))
    S, w = co.head_logits(q, k, 0.5)
    pairs = [(t, j) for t in range(6) for j in range(t + 1)]
    assert len(S) == len(pairs)
    ref = sorted((0.5 * float(q[t] @ k[j]), 1.0 / (t + 1)) for t, j in pairs)
    got = sorted(zip(S.tolist(), w.tolist()))
    np.testing.assert_allclose(np.array(got), np.array(ref), rtol=1e-14, atol=1e-14)


def test_total_weight_is_rows():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 4, 37, 8))
    k = rng.standard_normal((2, 2, 40, 8))
    res = co.calibration_logits(q, k, 37)
    for h in range(4):
        assert math.isclose(res[h][1].sum(), 2 * 37, rel_tol=1e-12)


def test_closed_form_density_and_constant():
    # one row of 4 logits (weight 1/4 each) and one of 1 logit (weight 1):
    # density at c is (count_row0(>= c) / 4 + [row1 >= c]) / 2
    S = np.array([1.0, 2.0, 3.0, 4.0, 10.0])
    w = np.array([0.25, 0.25, 0.25, 0.25, 1.0])
    assert co.density(S, w, 3.0) == (0.5 + 1.0) / 2
    assert co.density(S, w, 10.0) == 0.5
    assert co.exact_constant(S, w, 0.5) == 10.0
    assert co.exact_constant(S, w, 0.6) == 4.0
    assert co.exact_constant(S, w, 1.0) == 1.0


def test_constant_decreases_as_the_target_grows():
    rng = np.random.default_rng(2)
    S = rng.standard_normal(5000)
    w = rng.uniform(0.01, 1, 5000)
    cs = [co.exact_constant(S, w, p) for p in (0.05, 0.2, 0.38, 0.6, 0.9)]
    assert all(a >= b for a, b in zip(cs, cs[1:]))
    for p, c in zip((0.05, 0.2, 0.38, 0.6, 0.9), cs):
        assert co.density(S, w, c) >= p - 1e-12


def test_histogram_solver_within_one_bin():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 2, 200, 16))
    k = rng.standard_normal((1, 1, 200, 16))
    lo, hi, nb = -6.0, 6.0, 480
    for h, (S, w) in co.calibration_logits(q, k, 200).items():
        hist = co.histogram(S, w, lo, hi, nb)
        assert math.isclose(hist.sum(), 200.0, rel_tol=1e-12)
        for p in (0.1, 0.38, 0.7):
            c_hist = co.histogram_constant(hist, lo, hi, p)
            c_ex = co.exact_constant(S, w, p)
            assert abs(c_hist - c_ex) <= (hi - lo) / nb + 1e-12, (h, p, c_hist, c_ex)
