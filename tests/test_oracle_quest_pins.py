"""Pins of the coordinate-box (Quest) oracle and of the token-recall study:
strictness by brute force, closed forms (sign-constant queries pick one
extremum per coordinate; a one-key block bounds that key's own logit),
outward fp16 rounding against the exact extrema, and the recall counts of a
constructed case.  Mistakes such as max/min swapped, inward rounding or
recall counted over blocks instead of keys fail one of them."""
import numpy as np

from oracle import eta_quest_oracle as qo


def test_box_bound_is_strict_by_brute_force():
    rng = np.random.default_rng(0)
    for n in (1, 5, 64):
        k = rng.standard_normal((n, 32)) * rng.uniform(0.1, 4)
        lo, hi = qo.box_summary(k)
        for _ in range(20):
            q = rng.standard_normal(32)
            assert (k @ q).max() * 0.3 <= qo.box_scores(q, lo, hi, 0.3) + 1e-12


def test_closed_forms():
    k = np.array([[1.0, -2.0, 0.5], [3.0, 0.25, -1.0]])
    lo, hi = qo.box_summary(k)
    np.testing.assert_array_equal(lo.astype(np.float64), [1.0, -2.0, -1.0])
    np.testing.assert_array_equal(hi.astype(np.float64), [3.0, 0.25, 0.5])
    q = np.array([1.0, 2.0, 3.0])  # all positive: the maxima
    assert qo.box_scores(q, lo, hi, 1.0) == 3.0 + 0.5 + 1.5
    q = -q  # all negative: the minima
    assert qo.box_scores(q, lo, hi, 1.0) == -1.0 + 4.0 + 3.0
    one = np.array([[0.1, -0.7, 2.3]])
    lo1, hi1 = qo.box_summary(one)
    qv = np.array([0.4, -1.2, 0.9])
    assert qo.box_scores(qv, lo1, hi1, 1.0) >= float(one[0] @ qv)


def test_outward_rounding():
    x = np.array([0.1, -0.1, 1.0 / 3.0, 65000.0, -3.0])
    dn, up = qo._f16_down(x), qo._f16_up(x)
    assert np.all(dn.astype(np.float64) <= x) and np.all(up.astype(np.float64) >= x)
    # tight: the next fp16 value beyond is on the other side
    assert np.all(np.nextafter(dn, np.float16(np.inf)).astype(np.float64) > x)
    assert np.all(np.nextafter(up, np.float16(-np.inf)).astype(np.float64) < x)
    np.testing.assert_array_equal(dn[[4]], np.float16(-3.0))


def test_token_recall_counts():
    # 2 blocks of 2 keys; logits 1, 5 | 4, 0 with tau~ = 3: true keys 2 (one per block)
    q = np.array([1.0])
    K = np.array([[1.0], [5.0], [4.0], [0.0]])
    assert qo.token_recall(q, K, 4, 2, 3.0, 1.0, np.array([True, False])) == (2, 1)
    assert qo.token_recall(q, K, 4, 2, 3.0, 1.0, np.array([True, True])) == (2, 2)
    assert qo.token_recall(q, K, 3, 2, 3.0, 1.0, np.array([False, True])) == (2, 1)
