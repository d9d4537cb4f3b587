"""Write tests/golden/thresholds.json: per-head thresholds of the synthetic
decode workloads that target a GQA-union admitted density.

Calls only the CPU oracle (block summaries and block scores) and the seeded
input generator.  For each workload the same score quantile p is used for every
query head; p is bisected until the union density (always-loaded blocks
included) reaches the target.  Each head's effective threshold tau~ is then
placed in the middle of the widest gap between neighbouring block scores near
its quantile, so that no block score sits close to the threshold (fp32
evaluation on the device cannot flip a decision).

Learned mode stores b_tau = tau~ + a - w_tau . q (rounded to fp32);
calibrated mode stores c_tau = tau~ + a.

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
TARGETS = {"c2_single": 0.38, "c3_long": 0.38, "c4_max": 0.38}


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


def calibrate(name, seed=0):
    wl = workloads.make(name, seed)
    target = TARGETS[name]
    summary = oracle.summarize(wl.k, wl.seq_lens, wl.block_size)
    scores, screened_n = _scores(wl, summary)
    srt = {key: np.sort(val)[::-1] for key, val in scores.items()}

    def taus_for(p):
        return {key: _tau_for_count(s, int(round(p * len(s)))) for key, s in srt.items()}

    lo, hi = 0.0, 1.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if _union_density(wl, scores, screened_n, taus_for(mid)) < target:
            lo = mid
        else:
            hi = mid
    p = 0.5 * (lo + hi)
    taus = {}
    margins = {}
    for key, s in srt.items():
        n = len(s)
        k0 = int(round(p * n))
        w = max(2, int(0.01 * n))
        best_k, best_gap = k0, -1.0
        for k in range(max(1, k0 - w), min(n - 1, k0 + w) + 1):
            gap = s[k - 1] - s[k]
            if gap > best_gap:
                best_k, best_gap = k, gap
        taus[key] = _tau_for_count(s, best_k)
        margins[key] = best_gap / 2
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
    real_margin = min(float(np.min(np.abs(scores[key] - taus[key]))) for key in scores)
    entry["min_margin"] = real_margin
    entry["union_density"] = _union_density(wl, scores, screened_n, taus)
    head_dens = []
    for (i, h), sc in scores.items():
        ns, nb = screened_n[i]
        head_dens.append(((sc >= taus[(i, h)]).sum() + nb - ns) / nb)
    entry["mean_head_density"] = float(np.mean(head_dens))
    return entry


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
