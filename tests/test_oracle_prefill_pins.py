"""Pins of the causal forward (prefill) oracle against what the pages and plain
mathematics fix, each chosen so that a plausible mistake fails one of them:
a non-causal or off-by-one mask, the gate applied additively or to the wrong
row's threshold, a missing scale, R summed over the wrong keys, a wrong GQA
index, a natural/base-2 mix-up in the log-sum-exp.
"""
import math

import numpy as np
import torch

import oracle
from oracle import eta_prefill_oracle as po


def _inputs(seed, B=1, Hq=2, Hkv=1, T=37, d=16):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, d))
    return q, k, v


def _sdpa_causal(q, k, v, scale):
    """Library causal softmax attention (fp64 on the CPU), the sigma = 1 case."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale).numpy()


def _lse_causal(q, k, scale):
    S = scale * np.einsum("td,sd->ts", q, k)
    S = np.where(np.tril(np.ones_like(S, dtype=bool)), S, -np.inf)
    return np.logaddexp.reduce(S, axis=1)


def test_gate_open_is_plain_causal_attention():
    # tau~ far below every logit: sigma = 1, S~ = S, R_i = i + 1
    q, k, v = _inputs(1, Hq=4, Hkv=2, T=41, d=8)
    scale = 0.37
    r = po.prefill(q, k, v, 41, "calibrated", c_tau=np.full(4, -1e6), scale=scale, beta=5.0)
    for h in range(4):
        g = h // 2
        ref = _sdpa_causal(q[0, h], k[0, g], v[0, g], scale)
        np.testing.assert_allclose(r["out"][0, h], ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(r["lse"][0, h], _lse_causal(q[0, h], k[0, g], scale), rtol=1e-12)
        np.testing.assert_array_equal(r["gate_sum"][0, h], np.arange(1, 42, dtype=np.float64))


def test_beta_zero_halves_the_logits():
    # beta = 0: sigma = 1/2 exactly, S~ = S / 2: causal attention at half the scale
    q, k, v = _inputs(2, T=29, d=8)
    scale = 0.5
    tau = np.array([0.3, -2.0])
    r = po.prefill(q, k, v, 29, "calibrated", c_tau=tau, scale=scale, beta=0.0)
    for h in range(2):
        ref = _sdpa_causal(q[0, h], k[0, 0], v[0, 0], scale / 2)
        np.testing.assert_allclose(r["out"][0, h], ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(r["gate_sum"][0, h], np.arange(1, 30) / 2.0, rtol=0, atol=0)


def test_first_row_closed_form():
    # query 0 sees key 0 only: o_0 = v_0, L_0 = S~_00, R_0 = sigma_00
    q, k, v = _inputs(3, T=5, d=4)
    scale, beta, c = 0.8, 5.0, 0.25
    r = po.prefill(q, k, v, 5, "calibrated", c_tau=np.array([c, c]), scale=scale, beta=beta)
    for h in range(2):
        S = scale * float(q[0, h, 0] @ k[0, 0, 0])
        sig = 1.0 / (1.0 + math.exp(-beta * (S - c)))
        np.testing.assert_allclose(r["out"][0, h, 0], v[0, 0, 0], rtol=1e-15)
        assert r["lse"][0, h, 0] == S * sig or math.isclose(r["lse"][0, h, 0], S * sig, rel_tol=1e-15)
        assert math.isclose(r["gate_sum"][0, h, 0], sig, rel_tol=1e-15)


def test_brute_force_loop():
    # an explicit double loop over (query, key <= query)
    q, k, v = _inputs(4, T=11, d=6)
    scale, beta, a = 0.6, 3.0, 0.1
    w = np.random.default_rng(5).standard_normal((2, 6)) * 0.2
    b = np.array([0.2, -0.1])
    r = po.prefill(q, k, v, 11, "learned", w_tau=w, b_tau=b, scale=scale, beta=beta, offset_a=a)
    for h in range(2):
        for i in range(11):
            tau = float(w[h] @ q[0, h, i]) + b[h] - a
            logits, gates = [], []
            for j in range(i + 1):
                S = scale * float(q[0, h, i] @ k[0, 0, j])
                sg = 1.0 / (1.0 + math.exp(-beta * (S - tau)))
                logits.append(S * sg)
                gates.append(sg)
            m = max(logits)
            ws = [math.exp(x - m) for x in logits]
            o = sum(wj * v[0, 0, j] for j, wj in enumerate(ws)) / sum(ws)
            np.testing.assert_allclose(r["out"][0, h, i], o, rtol=1e-12, atol=1e-13)
            assert math.isclose(r["lse"][0, h, i], m + math.log(sum(ws)), rel_tol=1e-12, abs_tol=1e-12)
            assert math.isclose(r["gate_sum"][0, h, i], sum(gates), rel_tol=1e-12)


def test_last_row_matches_the_decode_oracle():
    # the last query row of the causal pass is a dense decode step of that query
    q, k, v = _inputs(6, Hq=4, Hkv=2, T=40, d=8)
    scale, beta, a = 0.35, 5.0, 0.4
    w = np.random.default_rng(7).standard_normal((4, 8)) * 0.1
    b = np.full(4, 0.5)
    r = po.prefill(q, k, v, 40, "learned", w_tau=w, b_tau=b, scale=scale, beta=beta, offset_a=a)
    block = 8
    for h in range(4):
        g = h // 2
        qt = q[0, h, 39]
        tau = oracle.threshold_learned(qt, w[h], b[h], a)
        o, lse = oracle.attend_head(qt, k[0, g], v[0, g], 40, block, np.ones(5, dtype=bool), tau, scale, beta)
        np.testing.assert_allclose(r["out"][0, h, 39], o, rtol=1e-12, atol=1e-13)
        assert math.isclose(r["lse"][0, h, 39], lse, rel_tol=1e-12)


def test_flop_count():
    # 4 d flops per causal (query, key) pair: T (T + 1) / 2 pairs per head
    assert po.prefill_flops(2, 3, 4, 8) == 4 * 8 * 10 * 2 * 3


def test_row_form_matches_whole_head_and_decode():
    # prefill_row(i) over keys 0..i is row i of the whole-head causal pass, and
    # at every i it is a dense decode step of q_i over a cache of i + 1 keys
    q, k, v = _inputs(8, Hq=1, Hkv=1, T=33, d=8)
    scale, beta = 0.4, 5.0
    tau = po.prefill_thresholds(q[0, 0], "calibrated", c_h=0.3)
    O, L, R = po.prefill_head(q[0, 0], k[0, 0], v[0, 0], tau, scale, beta)
    for i in (0, 1, 7, 8, 31, 32):
        o, lse, r = po.prefill_row(q[0, 0, i], k[0, 0, :i + 1], v[0, 0, :i + 1], tau[i], scale, beta)
        np.testing.assert_allclose(o, O[i], rtol=1e-12, atol=1e-13)
        assert math.isclose(lse, L[i], rel_tol=1e-12) and math.isclose(r, R[i], rel_tol=1e-12)
        nb = (i + 1 + 3) // 4
        o2, lse2 = oracle.attend_head(q[0, 0, i], k[0, 0], v[0, 0], i + 1, 4, np.ones(nb, dtype=bool), tau[i],
                                      scale, beta)
        np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
        assert math.isclose(lse, lse2, rel_tol=1e-12)
