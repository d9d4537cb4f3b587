"""Host-side check of the FMA-pipe 2^y of the causal forward kernel
(csrc/prefill_tc.cu, between the ETA_EXP2 markers).  Three pairs in eight of
the softmax weights 2^(x - m) are computed there with a Cody-Waite style
range reduction and a cubic for 2^f on [-1/2, 1/2], instead of the
special-function unit.  The block is compiled for the host with g++ (its
packed pair operations fall back to the scalar forms, which round each
element the same way) and compared with exp2 in long double:

* relative error at most 8e-5 wherever a weight can be (y in [-125, 8]: the
  lazy running max keeps y <= 8), including at integers and half-integers
  (the rounding of n) and across the exponent range;
* below that the result only has to be negligible next to the weights of
  order 1 it is summed with: it stays in [0, 2^-124];
* the cubic's own coefficients reach the fitted error bound and not much
  more: a wrong coefficient (a dropped or mis-scaled term) fails."""
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "learned_threshold_sparse_b200", "csrc", "prefill_tc.cu")

PRELUDE = r"""
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#define __host__
#define __device__
struct float2 { float x, y; };
inline float2 make_float2(float a, float b) { return float2{a, b}; }
using std::fmaf;
using std::fmaxf;
"""

DRIVER = r"""
int main() {
  float a, b;
  while (scanf("%f %f", &a, &b) == 2) {
    const float2 r = exp2_fma2(make_float2(a, b));
    printf("%.9e %.9e\n", r.x, r.y);
  }
  return 0;
}
"""


def _block(src=None):
    src = src if src is not None else open(SRC).read()
    m = re.search(r"// ETA_EXP2_BEGIN\n(.*?)// ETA_EXP2_END", src, flags=re.S)
    assert m, "exp2 block not found"
    return m.group(1).replace("__host__ __device__ inline", "inline")


def _build(tmp_path, name, block):
    prog = tmp_path / f"{name}.cpp"
    prog.write_text(PRELUDE + block + DRIVER)
    exe = tmp_path / name
    subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", str(prog), "-o", str(exe)], check=True)

    def run(y):
        y = np.asarray(y, dtype=np.float32)
        n = len(y)
        yp = np.append(y, np.float32(0)) if n % 2 else y
        text = "\n".join(f"{float(yp[i]):.9g} {float(yp[i + 1]):.9g}" for i in range(0, len(yp), 2)) + "\n"
        out = subprocess.run([str(exe)], input=text, capture_output=True, text=True, check=True).stdout
        return y, np.array(out.split(), dtype=np.float64)[:n]

    return run


@pytest.fixture(scope="module")
def exp2_fma(tmp_path_factory):
    return _build(tmp_path_factory.mktemp("exp2"), "exp2", _block())


def _rel_err(y, got):
    want = np.exp2(y.astype(np.longdouble))
    return np.abs((got.astype(np.longdouble) - want) / want).astype(np.float64)


def test_relative_error_over_the_weight_range(exp2_fma):
    rng = np.random.default_rng(0)
    y = np.concatenate([np.linspace(-125.0, 8.0, 40001), rng.uniform(-30.0, 8.0, 20000),
                        np.arange(-125, 9), np.arange(-125, 8) + 0.5, np.arange(-125, 8) - 0.5,
                        [0.0, -0.0, 1e-8, -1e-8, 8.0, 7.999999]]).astype(np.float32)
    y, got = exp2_fma(y)
    err = _rel_err(y, got)
    assert err.max() <= 8e-5, (float(err.max()), float(y[np.argmax(err)]))
    assert np.all(got > 0)


def test_far_below_the_range_is_negligible(exp2_fma):
    y = np.concatenate([np.linspace(-400.0, -125.0, 5001), [-126.0, -127.0, -1e30, -np.inf]]).astype(np.float32)
    y, got = exp2_fma(y)
    assert np.all(got >= 0) and np.all(got <= 2.0 ** -124)


def test_the_fit_is_tight(exp2_fma):
    # the equioscillating cubic reaches close to its bound somewhere
    y, got = exp2_fma(np.linspace(-4.0, 4.0, 80001).astype(np.float32))
    assert _rel_err(y, got).max() >= 6e-5


@pytest.mark.parametrize("old,new", [
    ("0.69326097f, 0.69326097f", "0.69314718f, 0.69314718f"),   # the Taylor ln 2 in place of the fitted one
    ("0.05517167f, 0.05517167f", "0.0f, 0.0f"),                 # the cubic term dropped
    ("(bits_of(t.x) << 23)", "(bits_of(t.x) << 22)"),           # the exponent field misplaced
])
def test_a_planted_mistake_fails(tmp_path, old, new):
    src = open(SRC).read()
    assert old in src
    run = _build(tmp_path, "bad", _block(src.replace(old, new)))
    y, got = run(np.linspace(-20.0, 8.0, 2001).astype(np.float32))
    assert _rel_err(y, got).max() > 8e-5


def _remez_cubic_for_exp2():
    """Cubic of least maximum relative error for 2^f on [-1/2, 1/2], by the
    Remez exchange: solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on n + 2 points,
    move the points to the extrema of the relative error, repeat."""
    a, b, n = -0.5, 0.5, 3
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n + 2)[::-1] / (n + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(30):
        y = 2.0 ** x
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * y[i]
        c = np.linalg.solve(A, y)[:n + 1]
        r = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        idx = [0] + [i for i in range(1, len(grid) - 1) if (r[i] - r[i - 1]) * (r[i + 1] - r[i]) <= 0] + [len(grid) - 1]
        sel = []
        for xi, ri in zip(grid[idx], r[idx]):
            if sel and np.sign(ri) == np.sign(sel[-1][1]):
                if abs(ri) > abs(sel[-1][1]):
                    sel[-1] = (xi, ri)
            else:
                sel.append((xi, ri))
        while len(sel) > n + 2:
            sel.pop(0 if abs(sel[0][1]) < abs(sel[-1][1]) else -1)
        x = np.array([s[0] for s in sel])
    return c, float(np.abs(r).max())


def test_coefficients_are_the_minimax_cubic():
    # the constants in the kernel are this fit rounded to fp32
    c, err = _remez_cubic_for_exp2()
    assert 7.4e-5 < err < 7.6e-5
    block = _block()
    m = re.findall(r"make_float2\(([0-9.]+)f, \1f\)", block)
    coeffs = sorted(float(v) for v in m if float(v) < 2.0)  # the four polynomial constants
    assert len(coeffs) == 4, coeffs
    np.testing.assert_allclose(sorted(c), coeffs, rtol=2e-7, atol=0)
