"""Write tests/golden/thresholds.json: per-head thresholds of the synthetic
decode workloads that target a GQA-union admitted density.

Calls only the CPU oracle (block summaries and block scores) and the seeded
input generator.  For the density-targeted workloads the same score quantile p
is used for every query head; p is bisected until the union density
(always-loaded blocks included) reaches the target.  Each head's effective
threshold tau~ is then placed in the middle of the gap between neighbouring
block scores that is nearest to its quantile among the gaps wide enough that
every block score stays at least MIN_MARGIN away from tau~ (a guard band: the
device evaluates the bound in fp32, whose rounding error on these workloads
is below 2e-5, so no decision can flip).  The batched workload draws its
per-head constants U[0.5, 2.0]; each is moved to the middle of the nearest
such gap of that head's scores over all sequences.

Learned mode stores b_tau = tau~ + a - w_tau . q (rounded to fp32);
calibrated mode stores c_tau = tau~ + a (rounded to fp32).  The margins are
measured again after the rounding.

Usage:  python tests/golden/make_thresholds.py [name ...]
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "thresholds.json")
TARGETS = {"c2_single": 0.38, "c3_long": 0.38, "c4_max": 0.38, "c5_batched": None}
MIN_MARGIN = 1e-4


def _scores(wl, summary):
    """scores[(i, h)] = block scores of the screened blocks; forced[(i, g)]."""
    G = wl.group
    out = {}
    screened_n = {}
    for i, T in enumerate(wl.seq_lens):
        nb = wl.n_blocks(i)
        screened, forced = oracle.screened_and_forced(nb, wl.n_local_blocks)
        screened_n[i] = (int(screened.sum()), nb)
        for h in range(wl.n_q_heads):
            g = h // G
            sc = oracle.block_scores(oracle.as_f64(wl.q[i, h]), summary["mu"][i, g, :nb],
                                     summary["sigma"][i, g, :nb], summary["max_norm"][i, g, :nb],
                                     wl.scale, wl.z)
            out[(i, h)] = sc[screened]
    return out, screened_n


def _tau_for_count(sorted_desc, k):
    """Threshold admitting exactly the k highest scores, midway in the gap."""
    n = len(sorted_desc)
    if k <= 0:
        return sorted_desc[0] + 1.0
    if k >= n:
        return sorted_desc[-1] - 1.0
    return 0.5 * (sorted_desc[k - 1] + sorted_desc[k])


def _guarded_tau(sorted_desc, near):
    """The middle of the gap between neighbouring scores (or beyond the
    extremes) nearest to `near` whose half-width is at least MIN_MARGIN."""
    s = sorted_desc
    cands = []
    if len(s) == 0:
        return near
    cands.append(s[0] + MIN_MARGIN)      # above every score
    cands.append(s[-1] - MIN_MARGIN)     # below every score
    gaps = s[:-1] - s[1:]
    ok = np.flatnonzero(gaps >= 2 * MIN_MARGIN)
    cands.extend(0.5 * (s[ok] + s[ok + 1]))
    cands = np.asarray(cands)
    return float(cands[np.argmin(np.abs(cands - near))])


def _union_density(wl, scores, screened_n, taus):
    G = wl.group
    tot = 0.0
    for i in range(wl.batch):
        ns, nb = screened_n[i]
        for g in range(wl.n_kv_heads):
            adm = np.zeros(ns, bool)
            for j in range(G):
                h = g * G + j
                adm |= scores[(i, h)] >= taus[(i, h)]
            tot += (adm.sum() + (nb - ns)) / nb
    return tot / (wl.batch * wl.n_kv_heads)


def _finish(entry, wl, scores, screened_n, taus):
    real_margin = min(float(np.min(np.abs(scores[key] - taus[key]))) for key in scores if len(scores[key]))
    entry["min_margin"] = real_margin
    assert real_margin >= MIN_MARGIN * 0.999, real_margin
    entry["union_density"] = _union_density(wl, scores, screened_n, taus)
    head_dens = []
    for (i, h), sc in scores.items():
        ns, nb = screened_n[i]
        head_dens.append(((sc >= taus[(i, h)]).sum() + nb - ns) / nb)
    entry["mean_head_density"] = float(np.mean(head_dens))
    return entry


def _place_constants(wl, scores, screened_n):
    """Calibrated constants drawn per head (the workload's own draw), each
    moved into the nearest guard-banded gap of that head's scores pooled over
    the batch (the constant is shared by every sequence)."""
    pooled = {}
    for (i, h), sc in scores.items():
        pooled.setdefault(h, []).append(sc)
    c32 = np.zeros(wl.n_q_heads, np.float32)
    for h in range(wl.n_q_heads):
        sd = np.sort(np.concatenate(pooled[h]))[::-1]
        tt = _guarded_tau(sd, float(wl.c_tau[h]) - wl.offset_a)
        c32[h] = np.float32(tt + wl.offset_a)
    taus = {(i, h): oracle.threshold_calibrated(c32[h], wl.offset_a) for (i, h) in scores}
    entry = {"drawn_c_tau": [float(x) for x in wl.c_tau], "c_tau": [float(x) for x in c32]}
    return _finish(entry, wl, scores, screened_n, taus)


def calibrate(name, seed=0):
    wl = workloads.make(name, seed, raw_thresholds=True)
    target = TARGETS[name]
    summary = oracle.summarize(wl.k, wl.seq_lens, wl.block_size)
    scores, screened_n = _scores(wl, summary)
    if target is None:
        return _place_constants(wl, scores, screened_n)
    srt = {key: np.sort(val)[::-1] for key, val in scores.items()}

    def taus_for(p):
        return {key: _guarded_tau(s, _tau_for_count(s, int(round(p * len(s))))) for key, s in srt.items()}

    lo, hi = 0.0, 1.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if _union_density(wl, scores, screened_n, taus_for(mid)) < target:
            lo = mid
        else:
            hi = mid
    p = 0.5 * (lo + hi)
    taus = taus_for(p)
    entry = {"target_union_density": target, "quantile": p}
    if wl.tau_mode == "learned":
        b = np.zeros(wl.n_q_heads, np.float64)
        for h in range(wl.n_q_heads):
            wq = float(oracle.as_f64(wl.w_tau[h]) @ oracle.as_f64(wl.q[0, h]))
            b[h] = taus[(0, h)] + wl.offset_a - wq
        b32 = b.astype(np.float32)
        entry["b_tau"] = [float(x) for x in b32]
        # margins after rounding b to fp32
        for h in range(wl.n_q_heads):
            tt = oracle.threshold_learned(oracle.as_f64(wl.q[0, h]), wl.w_tau[h], b32[h], wl.offset_a)
            taus[(0, h)] = tt
    else:
        c32 = np.array([taus[(0, h)] + wl.offset_a for h in range(wl.n_q_heads)], np.float32)
        entry["c_tau"] = [float(x) for x in c32]
        for h in range(wl.n_q_heads):
            taus[(0, h)] = oracle.threshold_calibrated(c32[h], wl.offset_a)
    return _finish(entry, wl, scores, screened_n, taus)


def main(names):
    table = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            table = json.load(f)
    table["_about"] = ("Per-head thresholds for the synthetic decode workloads; written by "
                       "tests/golden/make_thresholds.py from the CPU oracle's block scores.")
    for name in names:
        entry = calibrate(name, 0)
        table.setdefault(name, {})["seed0"] = entry
        print(name, {k: v for k, v in entry.items() if not isinstance(v, list)}, flush=True)
    with open(OUT, "w") as f:
        json.dump(table, f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1:] or list(TARGETS))
