"""Pins of the CPU oracle against what the ETA pages and plain mathematics fix.

Each test would fail under a plausible mistake in the oracle: a dropped term or
factor in the bound, a wrong sign, a transposed operand, a wrong GQA index, an
off-by-one in the always-loaded window, a wrong rescue, a broken merge.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ P9 gate

def test_gate_closed_forms():
    # S~ = S sigma(beta (S - tau~)): at S = tau~ the gate is 1/2.
    for tau in (-1.5, 0.0, 2.25):
        for beta in (1.0, 5.0):
            assert oracle.tempered_logits(tau, tau, beta) == pytest.approx(tau / 2, abs=0)
    # at S = 0 the tempered logit is 0 whatever the gate
    assert oracle.tempered_logits(0.0, 0.7, 5.0) == 0.0
    # beta enters multiplicatively: sigma(ln 3) = 3/4
    tau, beta = 0.3, 5.0
    S = tau + math.log(3.0) / beta
    assert oracle.tempered_logits(S, tau, beta) == pytest.approx(0.75 * S, rel=1e-14)
    # far above threshold S~ -> S; far below S~ -> 0 (the uniform floor)
    assert oracle.tempered_logits(40.0, 0.0, 5.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.tempered_logits(-3.0, 5.0, 5.0)) < 1e-16


def test_sigmoid_slope_golden():
    g = _golden("sigmoid_slope.json")
    for p in g["points"]:
        s = oracle.sigmoid(p["x"])
        deriv = float(s * (1.0 - s)) if p["x"] < 30 else float(math.exp(-p["x"]) * oracle.sigmoid(p["x"]) ** 2)
        assert deriv == pytest.approx(p["derivative_printed"], rel=p["rel_tol"])


# ------------------------------------------------------------ P5 summaries

@pytest.mark.parametrize("n,d", [(1, 4), (2, 8), (7, 64), (64, 128)])
def test_block_summary_matches_numpy(n, d):
    rng = np.random.default_rng(n * 1000 + d)
    k = (rng.standard_normal((n, d)) * rng.uniform(0.01, 3.0, size=d) + rng.uniform(-2, 2, size=d)).astype(np.float32)
    mu, sg, M = oracle.block_summary(k)
    assert mu.dtype == np.float16 and sg.dtype == np.float16 and M.dtype == np.float32
    np.testing.assert_array_equal(mu, np.mean(k.astype(np.float64), axis=0).astype(np.float16))
    np.testing.assert_array_equal(sg, np.std(k.astype(np.float64), axis=0, ddof=0).astype(np.float16))
    brute = max(np.linalg.norm(k[s].astype(np.float64) - mu.astype(np.float64)) for s in range(n))
    assert float(M) >= brute
    assert float(M) <= float(np.nextafter(np.float32(brute), np.float32(np.inf)))
    if n == 1:
        assert np.all(sg == 0)


def test_sequence_summary_tail_block():
    rng = np.random.default_rng(3)
    T, b, d = 200, 64, 8
    k = rng.standard_normal((T, d)).astype(np.float32)
    mu, sg, M = oracle.sequence_summary(k, T, b)
    assert mu.shape == (4, d)
    mu3, sg3, M3 = oracle.block_summary(k[192:200])
    np.testing.assert_array_equal(mu[3], mu3)
    np.testing.assert_array_equal(sg[3], sg3)
    assert M[3] == M3
    mu1, _, _ = oracle.block_summary(k[64:128])
    np.testing.assert_array_equal(mu[1], mu1)


@pytest.mark.parametrize("T,b,d,dtype", [(256, 64, 16, "bf16"), (200, 64, 8, "f32"), (130, 16, 32, "f32"),
                                         (512, 128, 128, "bf16"), (97, 1, 4, "f32"), (64, 64, 8, "f32")])
def test_sequence_summary_every_full_block(T, b, d, dtype):
    # Every block of the vectorised path (full blocks) and the tail against
    # library statistics of that block alone: numpy mean, numpy population
    # std (ddof = 0) and a brute-force per-row norm loop around the stored
    # fp16 centroid.  A sample std (ddof = 1), a spread around the rounded
    # centroid, or M measured from the unrounded mean each fail here.
    # Coordinates spread from 1e-3 to 4 around offsets up to 3: where the
    # spread is small next to the offset, the fp16 rounding of the centroid
    # moves a spread measured around it by more than a half ulp.
    rng = np.random.default_rng(T * 7 + b * 3 + d)
    spread = 10.0 ** rng.uniform(-3, 0.6, size=d)
    k = torch.from_numpy((rng.standard_normal((T, d)) * spread + rng.uniform(-3, 3, size=d)).astype(np.float32))
    if dtype == "bf16":
        k = k.to(torch.bfloat16)
    mu, sg, M = oracle.sequence_summary(k, T, b)
    kf = k.float().numpy().astype(np.float64)
    nb = (T + b - 1) // b
    assert mu.shape == (nb, d) and sg.shape == (nb, d) and M.shape == (nb,)
    for j in range(nb):
        rows = kf[j * b:min(T, (j + 1) * b)]
        np.testing.assert_array_equal(mu[j], np.mean(rows, axis=0).astype(np.float16), err_msg=f"block {j}")
        np.testing.assert_array_equal(sg[j], np.std(rows, axis=0, ddof=0).astype(np.float16), err_msg=f"block {j}")
        centre = [float(x) for x in mu[j].astype(np.float64)]
        brute = 0.0
        for r in rows:
            brute = max(brute, math.sqrt(sum((float(r[e]) - centre[e]) ** 2 for e in range(d))))
        # M is the smallest fp32 value at or above the exact norm
        assert float(M[j]) >= brute, f"block {j}"
        assert float(np.nextafter(M[j], np.float32(-np.inf))) < brute, f"block {j}"
    if T % b == 0 and b > 1:
        assert sg[-1].any()  # a full last block is not summarised as a 1-row block


def test_metadata_overhead_golden():
    g = _golden("metadata_overhead.json")
    rec = oracle.metadata_record_bytes(g["head_dim"])
    kv = 2 * g["block_size"] * g["head_dim"] * g["kv_elt_bytes"]
    assert round(100.0 * rec / kv, 1) == g["overhead_percent_printed"]
    assert round(100.0 * g["record_bytes_printed"] / kv, 1) == g["overhead_percent_printed"]
    assert rec == g["record_bytes_printed"] + 2


# ------------------------------------------------------------ bound shape

def test_score_identical_keys_is_exact_logit():
    # sigma = 0: the probabilistic half is 0, Score = scale <q, mu_hat>
    d = 16
    rng = np.random.default_rng(5)
    key = rng.standard_normal(d).astype(np.float32)
    q = rng.standard_normal(d).astype(np.float32)
    blk = np.repeat(key[None], 8, axis=0)
    mu, sg, M = oracle.block_summary(blk)
    assert np.all(sg == 0)
    scale = 0.25
    sc = oracle.block_scores(q, mu[None], sg[None], np.array([M]), scale, 2.0)
    assert sc[0] == pytest.approx(scale * float(q.astype(np.float64) @ mu.astype(np.float64)), rel=1e-15)


def test_score_two_key_closed_form():
    # keys mu +- delta e_0: sigma = delta on coordinate 0, M = delta
    mu = np.array([0.5, -1.0, 2.0, 0.25], np.float32)
    delta = 0.75
    blk = np.stack([mu + delta * np.eye(4, dtype=np.float32)[0], mu - delta * np.eye(4, dtype=np.float32)[0]])
    m_hat, s_hat, M = oracle.block_summary(blk)
    np.testing.assert_array_equal(m_hat.astype(np.float32), mu)
    np.testing.assert_array_equal(s_hat.astype(np.float32), np.array([delta, 0, 0, 0], np.float32))
    assert float(M) == delta
    q = np.array([1.0, 2.0, 2.0, 4.0])
    scale = 0.5
    centre = float(q @ mu)  # 0.5 - 2 + 4 + 1 = 3.5
    assert centre == 3.5
    # z = 2: min(||q|| M, z |q_0| sigma_0) = min(5 * .75, 2 * .75) = 1.5
    sc = oracle.block_scores(q, m_hat[None], s_hat[None], np.array([M]), scale, 2.0)
    assert sc[0] == pytest.approx(scale * (3.5 + 1.5), rel=1e-15)
    # z = 10: the geometric half (3.75) is tighter
    sc = oracle.block_scores(q, m_hat[None], s_hat[None], np.array([M]), scale, 10.0)
    assert sc[0] == pytest.approx(scale * (3.5 + 3.75), rel=1e-15)
    # z = inf: strict geometric bound
    sc = oracle.block_scores(q, m_hat[None], s_hat[None], np.array([M]), scale, math.inf)
    assert sc[0] == pytest.approx(scale * (3.5 + 3.75), rel=1e-15)
    # the spread term uses q_i^2 of the coordinate that carries sigma
    q2 = np.array([3.0, 0.0, 0.0, 4.0])  # ||q|| = 5, |q_0| = 3
    sc = oracle.block_scores(q2, m_hat[None], s_hat[None], np.array([M]), 1.0, 1.0)
    assert sc[0] == pytest.approx(float(q2 @ mu) + min(5 * delta, 3 * delta), rel=1e-15)


# ------------------------------------------------------ P1 strict bound

@pytest.mark.parametrize("d", [4, 8, 64])
@pytest.mark.parametrize("b", [1, 2, 4, 64])
def test_geometric_bound_never_underestimates(d, b):
    rng = np.random.default_rng(d * 100 + b)
    for trial in range(20):
        n = b if trial % 3 else max(1, b - 1)
        kind = trial % 4
        if kind == 0:
            k = rng.standard_normal((n, d))
        elif kind == 1:
            k = rng.uniform(-5, 5, (n, d)) * rng.uniform(0, 1, d)
        elif kind == 2:
            k = rng.standard_normal((n, d)) * 1e-3 + 7.0
        else:
            k = rng.standard_cauchy((n, d))
        k = k.astype(np.float32)
        q = rng.standard_normal(d) * rng.uniform(0.1, 10)
        mu, sg, M = oracle.block_summary(k)
        scale = 1.0 / math.sqrt(d)
        bound = oracle.block_scores(q, mu[None], sg[None], np.array([M]), scale, math.inf)[0]
        logits = scale * (k.astype(np.float64) @ q)
        assert bound >= logits.max()


def test_strict_mode_admits_every_significant_block():
    rng = np.random.default_rng(11)
    T, b, d = 40 * 16, 16, 8
    k = rng.standard_normal((T, d)).astype(np.float32)
    q = rng.standard_normal(d)
    mu, sg, M = oracle.sequence_summary(k, T, b)
    scale = 1.0 / math.sqrt(d)
    logits = scale * (k.astype(np.float64) @ q)
    tau = float(np.quantile(logits, 0.97))
    sc = oracle.block_scores(q, mu, sg, M, scale, math.inf)
    adm, _ = oracle.admit(sc, tau, T // b, -1)
    significant = logits.reshape(-1, b).max(axis=1) >= tau
    assert significant.any() and not significant.all()
    assert np.all(adm[significant])


# ---------------------------------------------- window, rescue, union

def test_forced_window_and_screened_set():
    screened, forced = oracle.screened_and_forced(10, 2)
    np.testing.assert_array_equal(np.flatnonzero(forced), [7, 8, 9])
    np.testing.assert_array_equal(np.flatnonzero(screened), np.arange(7))
    screened, forced = oracle.screened_and_forced(2, 2)
    assert forced.all() and not screened.any()
    screened, forced = oracle.screened_and_forced(5, -1)
    assert screened.all() and not forced.any()
    adm, resc = oracle.admit(np.zeros(10), 1e9, 10, 2)
    np.testing.assert_array_equal(np.flatnonzero(adm), [7, 8, 9])
    assert not resc


def test_rescue_admits_exactly_the_argmax():
    rng = np.random.default_rng(2)
    for _ in range(50):
        nb = int(rng.integers(1, 40))
        sc = rng.standard_normal(nb)
        adm, resc = oracle.admit(sc, 1e9, nb, -1)
        assert resc and adm.sum() == 1 and adm[int(np.argmax(sc))]
    # ties go to the lowest index
    adm, _ = oracle.admit(np.array([0.0, 3.0, 1.0, 3.0]), 10.0, 4, -1)
    np.testing.assert_array_equal(np.flatnonzero(adm), [1])
    # nothing to rescue in an empty sequence
    adm, resc = oracle.admit(np.zeros(0), 0.0, 0, -1)
    assert adm.size == 0 and not resc


def test_gqa_grouping_and_union():
    wl = workloads.custom(seed=1, batch=1, n_q_heads=4, n_kv_heads=2, head_dim=8,
                          block_size=4, seq_lens=[37], dtype=workloads.F32,
                          tau_mode=workloads.TAU_LEARNED, tau_bias=1e9)
    v = wl.v.clone()
    v[0, 0] = 1.0
    v[0, 1] = -1.0
    r = oracle.decode(wl.q, wl.k, v, wl.seq_lens, wl.block_size, "learned",
                      wl.w_tau, wl.b_tau, n_local_blocks=2)
    np.testing.assert_allclose(r["o"][0, :2], 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["o"][0, 2:], -1.0, rtol=0, atol=1e-15)
    # union = OR of the group's admitted sets, mask bit j for head g*G + j
    wl2 = workloads.custom(seed=2, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=16,
                           block_size=8, seq_lens=[200, 77], dtype=workloads.F32,
                           tau_mode=workloads.TAU_LEARNED, tau_bias=1.2, tau_std=1.0)
    r = oracle.decode(wl2.q, wl2.k, wl2.v, wl2.seq_lens, 8, "learned", wl2.w_tau, wl2.b_tau)
    for i in range(2):
        for g in range(2):
            heads = r["admitted"][i, 4 * g:4 * g + 4]
            np.testing.assert_array_equal(r["union"][i, g], heads.any(axis=0))
            for j in range(4):
                np.testing.assert_array_equal((r["union_mask"][i, g] >> j) & 1, heads[j])


# ------------------------------------------------ P2, P3 special cases

def _sdpa(q, K, V, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], scale=scale)
    return out[0, 0, 0].numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_very_low_threshold_screen_off_is_plain_attention(seed):
    wl = workloads.custom(seed=seed, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=16,
                          block_size=8, seq_lens=[53, 8], dtype=workloads.F32,
                          tau_mode=workloads.TAU_LEARNED, tau_bias=-1e9)
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, 8, "learned", wl.w_tau, wl.b_tau,
                      scale=wl.scale, screen_enabled=False)
    for i, T in enumerate(wl.seq_lens):
        for h in range(4):
            K = oracle.as_f64(wl.k[i, h // 2, :T])
            V = oracle.as_f64(wl.v[i, h // 2, :T])
            ref = _sdpa(oracle.as_f64(wl.q[i, h]), K, V, wl.scale)
            np.testing.assert_allclose(r["o"][i, h], ref, rtol=0, atol=1e-13)
            lse = math.log(np.exp(wl.scale * (K @ oracle.as_f64(wl.q[i, h]))).sum())
            assert r["lse"][i, h] == pytest.approx(lse, rel=1e-13)
    assert np.all(r["admitted_count"][0] == 7) and np.all(r["admitted_count"][1] == 1)


def test_very_high_threshold_is_uniform_floor_over_window():
    wl = workloads.custom(seed=4, batch=1, n_q_heads=2, n_kv_heads=1, head_dim=8,
                          block_size=16, seq_lens=[150], dtype=workloads.F32,
                          tau_mode=workloads.TAU_LEARNED, tau_bias=1e9)
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, 16, "learned", wl.w_tau, wl.b_tau,
                      n_local_blocks=2)
    # nb = 10, forced blocks 7..9 = tokens 112..149, all weights e^0 = 1
    V = oracle.as_f64(wl.v[0, 0])
    for h in range(2):
        np.testing.assert_allclose(r["o"][0, h], V[112:150].mean(axis=0), rtol=0, atol=1e-14)
        assert r["lse"][0, h] == pytest.approx(math.log(38), rel=1e-14)
    # the screen off, same threshold: mean over the whole context
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, 16, "learned", wl.w_tau, wl.b_tau,
                      screen_enabled=False)
    np.testing.assert_allclose(r["o"][0, 0], V[:150].mean(axis=0), rtol=0, atol=1e-14)


# -------------------------------------------------------- P4 merge

@pytest.mark.parametrize("chunk", [1, 2, 3, 7])
def test_split_merge_is_associative(chunk):
    rng = np.random.default_rng(chunk)
    T, b, d = 300, 16, 32
    K = rng.standard_normal((T, d)) * 2
    V = rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    nb = (T + b - 1) // b
    adm = rng.uniform(size=nb) < 0.6
    adm[-1] = True
    o1, l1 = oracle.attend_head(q, K, V, T, b, adm, 0.4, 1 / math.sqrt(d), 5.0)
    o2, l2 = oracle.attend_head_chunked(q, K, V, T, b, adm, 0.4, 1 / math.sqrt(d), 5.0, chunk)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    assert l1 == pytest.approx(l2, rel=1e-13)
    # an empty partial merges as the identity
    part = oracle.partial_state(q, K, V, 0.4, 0.1, 5.0, np.zeros(T, bool))
    assert part[1] == -math.inf and part[2] == 0.0
    full = oracle.partial_state(q, K, V, 0.4, 0.1, 5.0, np.ones(T, bool))
    o3, _ = oracle.combine_partials([part, full, part])
    o4, _ = oracle.combine_partials([full])
    np.testing.assert_array_equal(o3, o4)


# ---------------------------------------------------------- P6, P8

def test_tiny_planted_blocks_admitted():
    wl = workloads.tiny(0)
    for z in (2.0, math.inf):
        r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, wl.block_size, "learned",
                          wl.w_tau, wl.b_tau, z=z)
        for (i, h), blocks in wl.planted.items():
            assert r["admitted"][i, h, blocks].all()
            # planted logits ~ 2 ||q||^2 / sqrt(d) = 16 dominate the output's weight
            assert r["scores"][i, h, blocks].min() > 10


def test_densities_are_counts_over_blocks():
    res = {
        "admitted": np.zeros((1, 2, 5), bool),
        "union": np.zeros((1, 1, 5), bool),
    }
    res["admitted"][0, 0, [0, 4]] = True
    res["admitted"][0, 1, [1, 4]] = True
    res["union"][0, 0] = res["admitted"][0].any(axis=0)
    res["admitted_count"] = res["admitted"].sum(axis=2)
    res["union_count"] = res["union"].sum(axis=2)
    dd = oracle.densities(res, [70], 16)  # nb = 5, last block has 6 tokens
    np.testing.assert_allclose(dd["head"][0], [2 / 5, 2 / 5])
    np.testing.assert_allclose(dd["union"][0], [3 / 5])
    np.testing.assert_allclose(dd["token_fraction"][0], [22 / 70, 22 / 70])


def test_start_dense_init_admits_everything():
    g = _golden("start_dense.json")
    wl = workloads.custom(seed=9, batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64,
                          block_size=64, seq_lens=[4096], dtype=workloads.BF16,
                          tau_mode=workloads.TAU_LEARNED, tau_bias=g["b_tau"], tau_std=0.0)
    assert np.all(wl.w_tau == g["w_tau"])
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, 64, "learned", wl.w_tau, wl.b_tau)
    dd = oracle.densities(r, wl.seq_lens, 64)
    assert np.all(dd["head"] == g["expected_density"])


def test_threshold_forms():
    q = np.array([3.0, 1.0, -2.0])
    w = np.array([2.0, 0.0, 0.5])
    assert oracle.threshold_learned(q, w, 0.5, 0.0) == 6.5 - 1.0 + 0.0
    assert oracle.threshold_learned(q, w, 0.5, 0.4) == pytest.approx(5.5 - 0.4)
    assert oracle.threshold_calibrated(1.25, 0.4) == pytest.approx(0.85)


def test_fp32_round_up():
    x = np.array([1.0, 1.0 + 1e-12, 0.1, 3.0 - 1e-13])
    r = oracle.fp32_round_up(x)
    assert np.all(r.astype(np.float64) >= x)
    assert r[0] == 1.0 and r[1] == np.nextafter(np.float32(1.0), np.float32(2.0))
