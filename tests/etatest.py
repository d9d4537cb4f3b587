"""Helpers shared by the GPU parity tests: run a workload through the CUDA
library (C ABI via the binding) and compare it with the CPU oracle.

Comparison rules (written out here so every test uses the same ones):
  * admitted block sets, per query head and per GQA union, must be identical;
    the one allowance is a block whose oracle margin |Score - tau~| is below
    the rounding error bound of the device's fp32 evaluation of the bound and
    the threshold (screen_error_bound: the device decides in fp32, Appendix
    F.2 of the ETA pages, so either decision is correct there).  For such a
    head the oracle's output is taken for the admitted set the device chose,
    which must differ from the oracle's own set only on those blocks.  With
    strict=True (the guard-banded workloads) no allowance is made at all.
  * outputs within OUT_TOL[dtype] max-abs, lse within LSE_TOL[dtype].
  * block metadata bit-exact: the device evaluates the statistics in float64
    and rounds once, like the oracle; a stored value may differ only where the
    oracle's float64 statistic lies within a float64 hair of a rounding
    boundary of the storage format (near_boundary).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import learned_threshold_sparse_b200 as eta
import oracle

U32 = 2.0 ** -24   # unit roundoff of fp32
HAIR = 2.0 ** -44  # relative distance of a float64 statistic from a rounding boundary that float64 noise can cross
OUT_TOL = {"bf16": 2e-2, "f32": 1e-4}
LSE_TOL = {"bf16": 2e-3, "f32": 1e-4}


def upload(wl, device="cuda"):
    d = {
        "q": wl.q.to(device),
        "k": wl.k.to(device),
        "v": wl.v.to(device),
        "seq": torch.tensor(wl.seq_lens, dtype=torch.int32, device=device),
    }
    for name in ("w_tau", "b_tau", "c_tau"):
        val = getattr(wl, name)
        d[name] = None if val is None else torch.from_numpy(np.ascontiguousarray(val, np.float32)).to(device)
    return d


def gpu_summary(wl, t):
    summ = eta.alloc_summary(wl.batch, wl.n_kv_heads, wl.max_ctx, wl.head_dim, wl.block_size)
    first = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    eta.eta_block_summary_update(t["k"], t["v"], t["seq"], summ, wl.block_size, first, wl.nb_max,
                                 wl.n_q_heads)
    return summ


def gpu_decode(wl, t=None, summ=None, attend_impl=eta.ETA_ATTEND_AUTO, **over):
    """Run one decode step on the device; returns host numpy arrays."""
    if t is None:
        t = upload(wl)
    if summ is None:
        summ = gpu_summary(wl, t)
    p = dict(scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
             n_local_blocks=wl.n_local_blocks, screen_enabled=wl.screen_enabled)
    p.update(over)
    res = eta.decode(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, wl.tau_mode,
                     w_tau=t["w_tau"], b_tau=t["b_tau"], c_tau=t["c_tau"], attend_impl=attend_impl,
                     selection=True, **p)
    torch.cuda.synchronize()
    status = eta.eta_read_device_status(res["workspace"])
    out = {k: v.float().cpu().numpy() if k == "out" else v.cpu().numpy()
           for k, v in res.items() if k != "workspace"}
    out["status"] = status
    out["summary"] = {k: v.cpu().numpy() for k, v in summ.items()}
    return out


def oracle_decode(wl, **over):
    p = dict(scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
             n_local_blocks=wl.n_local_blocks, screen_enabled=wl.screen_enabled)
    p.update(over)
    return oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, wl.block_size, wl.tau_mode,
                         w_tau=wl.w_tau, b_tau=wl.b_tau, c_tau=wl.c_tau, **p)


def screen_error_bound(wl, r, i, h, nb):
    """Per-block bound on |device (Score - tau~) - exact (Score - tau~)| for
    query head h of sequence i: the device evaluates the block bound and the
    threshold in fp32 (dot products over d split across lanes, then a
    butterfly: at most ~10 roundings deep), so the error is a few units of
    fp32 roundoff of the magnitudes summed.  32 u per summed magnitude keeps a
    wide safety factor."""
    G = wl.group
    g = h // G
    q = oracle.as_f64(wl.q[i, h])
    aq = np.abs(q)
    sc = wl.scale
    if "kmin" in r:  # the coordinate-box screen
        lo = np.asarray(r["kmin"][i, g, :nb], np.float64)
        hi = np.asarray(r["kmax"][i, g, :nb], np.float64)
        mag = np.maximum(np.abs(lo), np.abs(hi)) @ aq
        err = sc * 32 * U32 * mag
    else:
        mu = np.asarray(r["mu"][i, g, :nb], np.float64)
        sg = np.asarray(r["sigma"][i, g, :nb], np.float64)
        mm = np.asarray(r["max_norm"][i, g, :nb], np.float64)
        dot_mag = np.abs(mu) @ aq
        geo = np.sqrt(q @ q) * mm
        prob = (wl.z if np.isfinite(wl.z) else 0.0) * np.sqrt((sg * sg) @ (q * q))
        err = sc * 32 * U32 * (dot_mag + np.maximum(geo, prob))
    if wl.tau_mode == "learned":
        tau_mag = float(np.abs(oracle.as_f64(wl.w_tau[h])) @ aq) + abs(float(wl.b_tau[h])) + abs(wl.offset_a)
    else:
        tau_mag = abs(float(wl.c_tau[h])) + abs(wl.offset_a)
    return err + 32 * U32 * tau_mag


def near_boundary(x, encode):
    """True where the float64 value x lies within HAIR (relative) of a
    rounding boundary of `encode` (a function from float64 values to stored
    codes/values): nudging x by that much up or down changes its encoding."""
    x = np.asarray(x, np.float64)
    lo = encode(x - np.abs(x) * HAIR)
    hi = encode(x + np.abs(x) * HAIR)
    return np.asarray(lo != hi)


def assert_bits_equal(got, ref, exact_stat, encode, what):
    """got == ref element by element, except where the exact statistic sits
    within a float64 hair of the storage format's rounding boundary; returns
    the number of such excused elements (printed)."""
    got = np.asarray(got)
    ref = np.asarray(ref)
    diff = got != ref
    if not diff.any():
        return 0
    excused = diff & near_boundary(exact_stat, encode)
    bad = diff & ~excused
    assert not bad.any(), f"{what}: {int(bad.sum())} stored values differ at {np.argwhere(bad)[:5].tolist()}"
    n = int(excused.sum())
    print(f"{what}: {n} stored values differ next to a rounding boundary")
    assert n <= max(1, got.size // 100000)
    return n


def _fp16_encode(x):
    return np.asarray(x, np.float64).astype(np.float16)


def assert_summary_bit_exact(wl, got, ref, blocks=None):
    """Device fp16 metadata (got: numpy arrays) equals the oracle's (ref)
    value for value; M equal or one fp32 step above (the device inflates its
    float64 distance by 2^-47 before rounding up).  `blocks(i)` restricts the
    check to some blocks of sequence i.  Returns the number of excused
    near-boundary values."""
    n_exc = 0
    for i, T in enumerate(wl.seq_lens):
        nb = wl.n_blocks(i)
        js = list(range(nb)) if blocks is None else list(blocks(i))
        if not js:
            continue
        for g in range(wl.n_kv_heads):
            K = oracle.as_f64(wl.k[i, g, :T])
            rows = [K[j * wl.block_size:min(T, (j + 1) * wl.block_size)] for j in js]
            mean = np.stack([r_.mean(axis=0) for r_ in rows])
            std = np.stack([r_.std(axis=0) for r_ in rows])
            n_exc += assert_bits_equal(got["mu"][i, g, js], ref["mu"][i, g, js], mean, _fp16_encode,
                                       f"mu seq {i} kv {g}")
            n_exc += assert_bits_equal(got["sigma"][i, g, js], ref["sigma"][i, g, js], std, _fp16_encode,
                                       f"sigma seq {i} kv {g}")
            m_g = got["max_norm"][i, g, js].astype(np.float32)
            m_r = ref["max_norm"][i, g, js].astype(np.float32)
            up = np.nextafter(m_r, np.float32(np.inf))
            assert np.all((m_g == m_r) | (m_g == up)), f"max_norm seq {i} kv {g}"
            # M bounds every key's distance to the device's own centroid
            mu_g = got["mu"][i, g, js].astype(np.float64)
            for x, j in enumerate(js):
                assert np.sqrt(((rows[x] - mu_g[x]) ** 2).sum(axis=1)).max() <= float(m_g[x])
    return n_exc


def oracle_screen_on(wl, summary, r):
    """The oracle's screen (block_scores, admit, union) evaluated on the given
    metadata (e.g. the device's own), with the oracle's thresholds r["tau_tilde"].
    Returns the per-head admitted sets [B, Hq, nbmax]."""
    G = wl.group
    adm = np.zeros((wl.batch, wl.n_q_heads, wl.nb_max), bool)
    for i in range(wl.batch):
        nb = wl.n_blocks(i)
        for h in range(wl.n_q_heads):
            g = h // G
            sc = oracle.block_scores(oracle.as_f64(wl.q[i, h]), summary["mu"][i, g, :nb], summary["sigma"][i, g, :nb],
                                     summary["max_norm"][i, g, :nb], wl.scale, wl.z) if nb else np.zeros(0)
            a, _ = oracle.admit(sc, r["tau_tilde"][i, h], nb, wl.n_local_blocks, wl.screen_enabled)
            adm[i, h, :nb] = a
    return adm


def gpu_admitted(wl, g):
    """Per-head admitted sets [B, Hq, nbmax] from the exported union list/mask."""
    B, Hq, G = wl.batch, wl.n_q_heads, wl.group
    adm = np.zeros((B, Hq, wl.nb_max), bool)
    for i in range(B):
        for kv in range(wl.n_kv_heads):
            n = int(g["union_count"][i, kv])
            ids = g["union_list"][i, kv, :n]
            msk = g["union_mask"][i, kv, :n].astype(np.int64)
            assert np.all(np.diff(ids) > 0), "union list not ascending"
            assert np.all(msk != 0), "listed block with an empty head mask"
            assert np.all(g["union_list"][i, kv, n:] == -1)
            for j in range(G):
                adm[i, kv * G + j, ids[(msk >> j) & 1 == 1]] = True
    return adm


def compare(wl, g, r, out_tol=None, lse_tol=None, heads=None, strict=False):
    """Assert device results g equal oracle results r under the rules above.
    Returns the number of (head, block) decisions that fell in the band (0
    whenever strict)."""
    dt = wl.dtype
    out_tol = OUT_TOL[dt] if out_tol is None else out_tol
    lse_tol = LSE_TOL[dt] if lse_tol is None else lse_tol
    assert g["status"] == eta.ETA_OK, eta.eta_status_string(g["status"])
    adm_g = gpu_admitted(wl, g)
    G = wl.group
    n_amb = 0
    for i, T in enumerate(wl.seq_lens):
        nb = wl.n_blocks(i)
        for h in range(wl.n_q_heads):
            if heads is not None and (i, h) not in heads:
                continue
            a_o = r["admitted"][i, h, :nb]
            a_g = adm_g[i, h, :nb]
            assert not adm_g[i, h, nb:].any()
            diff = a_o != a_g
            if strict:
                assert not diff.any(), (f"seq {i} head {h}: admitted sets differ at blocks {np.flatnonzero(diff)[:10]}")
            margin = r["scores"][i, h, :nb] - r["tau_tilde"][i, h]
            bound = screen_error_bound(wl, r, i, h, nb) if nb else np.zeros(0)
            band = np.abs(np.nan_to_num(margin, nan=np.inf)) < bound
            assert not np.any(diff & ~band), (
                f"seq {i} head {h}: admitted sets differ outside the fp32 band at blocks "
                f"{np.flatnonzero(diff & ~band)[:10]} (margins {margin[diff & ~band][:10]})")
            o_ref, lse_ref = r["o"][i, h], r["lse"][i, h]
            if diff.any():
                n_amb += int(diff.sum())
                K = oracle.as_f64(wl.k[i, h // G, :T])
                V = oracle.as_f64(wl.v[i, h // G, :T])
                o_ref, lse_ref = oracle.attend_head(oracle.as_f64(wl.q[i, h]), K, V, T, wl.block_size, a_g,
                                                    r["tau_tilde"][i, h], wl.scale, wl.beta)
            err = np.abs(g["out"][i, h] - o_ref).max() if T > 0 else np.abs(g["out"][i, h]).max()
            assert err <= out_tol, f"seq {i} head {h}: out max-abs error {err} > {out_tol}"
            if T > 0:
                assert abs(g["lse"][i, h] - lse_ref) <= lse_tol * max(1.0, abs(lse_ref)), (
                    f"seq {i} head {h}: lse {g['lse'][i, h]} vs {lse_ref}")
            else:
                assert g["lse"][i, h] == -math.inf
    # integer counts: per head and per union, exact against the device's own sets
    np.testing.assert_array_equal(g["admitted_count"], adm_g.sum(axis=2))
    np.testing.assert_array_equal(g["union_count"],
                                  adm_g.reshape(wl.batch, wl.n_kv_heads, G, -1).any(axis=2).sum(axis=2))
    if n_amb == 0 and heads is None:
        np.testing.assert_array_equal(g["admitted_count"], r["admitted_count"])
        np.testing.assert_array_equal(g["union_count"], r["union_count"])
    return n_amb


def min_margin_over_bound(wl, r):
    """Smallest |Score - tau~| / screen_error_bound over every screened
    (sequence, head, block): above 1 means no decision can depend on the fp32
    evaluation."""
    best = math.inf
    for i in range(wl.batch):
        nb = wl.n_blocks(i)
        if nb == 0:
            continue
        for h in range(wl.n_q_heads):
            m = np.abs(r["scores"][i, h, :nb] - r["tau_tilde"][i, h])
            ok = np.isfinite(m)
            if ok.any():
                best = min(best, float((m[ok] / screen_error_bound(wl, r, i, h, nb)[ok]).min()))
    return best
