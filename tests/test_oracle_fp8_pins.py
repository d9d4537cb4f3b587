"""Pins of the FP8 metadata oracle: the e4m3 rounding against a brute-force
nearest-value search over all codes (fp32 inputs, and float64 points next to
every rounding boundary), closed forms of the scale and of a constant block,
codes nearest to numpy's mean and population std, the strict geometric bound
by brute force, and the distance of the dequantised statistics from the exact
ones (at most half an e4m3 step).
A plausible mistake (truncation instead of rounding, a scale off by the max,
M measured from the fp32 instead of the dequantised centroid, a spread from
the wrong mean) fails one of them."""
import math

import numpy as np
import pytest
import torch

from oracle import eta_fp8_oracle as fo


def _values():
    codes = np.arange(256, dtype=np.uint8)
    vals = fo.e4m3_decode(codes).astype(np.float64)
    finite = np.isfinite(vals)
    return codes[finite], vals[finite]


def test_e4m3_known_codes():
    enc = fo.e4m3_encode(np.array([0.0, 1.0, -2.0, 448.0, 2.0 ** -9, 1e6, -1e6, 0.875], np.float32))
    np.testing.assert_array_equal(enc, np.array([0x00, 0x38, 0xC0, 0x7E, 0x01, 0x7E, 0xFE, 0x36], np.uint8))
    np.testing.assert_array_equal(fo.e4m3_decode(np.array([0x38, 0x7E, 0x01, 0x08], np.uint8)),
                                  np.array([1.0, 448.0, 2.0 ** -9, 2.0 ** -6], np.float32))


def test_e4m3_rounding_is_nearest_even_by_brute_force():
    codes, vals = _values()
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.uniform(-2, 2, 20000),
                        (vals[:-1] + np.diff(vals) / 2)[np.diff(vals) > 0]]).astype(np.float32)
    got = fo.e4m3_encode(x)
    for xi, gi in zip(x.astype(np.float64), got):
        dist = np.abs(vals - xi)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:  # tie: the even mantissa (even code) wins; +0 / -0 both fine for 0
            best = [b for b in best if codes[b] % 2 == 0] or best
        assert fo.e4m3_decode(np.array([gi], np.uint8))[0] == vals[best[0]], (xi, gi)


def _nearest_by_search(x):
    """Brute force: the e4m3 code whose value is nearest to each float64 x
    (ties to the even code), saturating at +-448."""
    codes, vals = _values()
    out = np.empty(len(x), np.uint8)
    for n, xi in enumerate(np.asarray(x, np.float64)):
        xs = min(max(xi, -448.0), 448.0)
        dist = np.abs(vals - xs)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:
            best = [b for b in best if codes[b] % 2 == 0] or best
        c = int(codes[best[0]])
        if vals[best[0]] == 0.0:  # zero takes the value's sign
            c = 0x80 if np.signbit(xi) else 0x00
        out[n] = c
    return out


def test_e4m3_rounding_at_float64_points_next_to_every_boundary():
    # every rounding boundary (midpoint of neighbouring values), the points a
    # hair above and below it in float64, and the saturation region
    codes, vals = _values()
    pos = np.unique(vals[vals >= 0])
    mids = (pos[:-1] + pos[1:]) / 2
    eps = 2.0 ** -40
    x = np.concatenate([mids, mids * (1 + eps), mids * (1 - eps), pos, [448.0 * (1 + eps), 460.0, 470.0, 1e300]])
    x = np.concatenate([x, -x, [-1e-300, -0.0, 0.0]])
    np.testing.assert_array_equal(fo.e4m3_encode(x), _nearest_by_search(x))


def test_scale_maps_the_largest_coordinate_to_448():
    rng = np.random.default_rng(1)
    k = rng.standard_normal((64, 16)).astype(np.float32)
    s = fo.block_summary_fp8(k)
    mean = np.mean(k.astype(np.float64), axis=0)
    assert s["mu_scale"] == np.float32(np.abs(mean).max() / 448.0)
    assert np.abs(fo.e4m3_decode(s["mu_code"])).max() == 448.0
    std = np.std(k.astype(np.float64), axis=0, ddof=0)
    assert s["sigma_scale"] == np.float32(std.max() / 448.0)


@pytest.mark.parametrize("n,d,dtype", [(64, 128, "bf16"), (7, 32, "f32"), (128, 64, "bf16"), (1, 16, "f32")])
def test_codes_are_nearest_to_the_exact_statistics(n, d, dtype):
    # codes of the centroid and the spread are the e4m3 values nearest to
    # numpy's mean and population std divided by the block's scale
    rng = np.random.default_rng(n + d)
    k = torch.from_numpy((rng.standard_normal((n, d)) * 10.0 ** rng.uniform(-2, 1, d)
                          + rng.uniform(-2, 2, d)).astype(np.float32))
    if dtype == "bf16":
        k = k.to(torch.bfloat16)
    kf = k.float().numpy().astype(np.float64)
    s = fo.block_summary_fp8(k)
    for name, val in (("mu", np.mean(kf, axis=0)), ("sigma", np.std(kf, axis=0, ddof=0))):
        scl = float(s[name + "_scale"])
        np.testing.assert_array_equal(s[name + "_code"], _nearest_by_search(val / scl), err_msg=name)
        np.testing.assert_array_equal(s[name], fo.e4m3_decode(s[name + "_code"]).astype(np.float64) * scl)


def test_constant_block():
    # 16 equal rows of short dyadic values: every fp32 sum is exact, so the
    # mean is the row and the spread is exactly zero
    row = (np.arange(-12, 12) / 4.0).astype(np.float32)
    k = np.tile(row, (16, 1))
    s = fo.block_summary_fp8(k)
    assert np.all(s["sigma_code"] == 0) and s["sigma_scale"] == 1.0
    np.testing.assert_allclose(s["mu"], row, rtol=2.0 ** -4, atol=0)
    exact = math.sqrt(float(((row.astype(np.float64) - s["mu"].astype(np.float64)) ** 2).sum()))
    assert float(s["max_norm"]) >= exact and float(np.nextafter(s["max_norm"], np.float32(0))) < exact


def test_geometric_half_is_a_true_bound_by_brute_force():
    rng = np.random.default_rng(2)
    for n in (1, 7, 64, 128):
        k = (rng.standard_normal((n, 24)) * rng.uniform(0.1, 5)).astype(np.float32)
        s = fo.block_summary_fp8(k)
        norms = np.sqrt(((k.astype(np.float64) - s["mu"].astype(np.float64)) ** 2).sum(axis=1))
        assert norms.max() <= float(s["max_norm"])
        # and for any query q: q.k <= q.mu~ + ||q|| M
        q = rng.standard_normal(24)
        assert (k.astype(np.float64) @ q).max() <= q @ s["mu"].astype(np.float64) + np.linalg.norm(q) * float(s["max_norm"]) + 1e-9


def test_dequantised_statistics_within_half_a_step():
    rng = np.random.default_rng(3)
    k = (rng.standard_normal((50, 40)) * 2 + 0.5).astype(np.float32)
    s = fo.block_summary_fp8(k)
    mean = k.astype(np.float64).mean(axis=0)
    std = k.astype(np.float64).std(axis=0)
    # e4m3 keeps 3 fraction bits: half a step is 2^-4 relative, plus half the
    # subnormal step 2^-10 of the scaled range
    tol_mu = 2.0 ** -4 * np.abs(mean) + 2.0 ** -10 * float(s["mu_scale"])
    tol_sd = 2.0 ** -4 * std + 2.0 ** -10 * float(s["sigma_scale"])
    assert np.all(np.abs(s["mu"] - mean) <= tol_mu)
    assert np.all(np.abs(s["sigma"] - std) <= tol_sd)
