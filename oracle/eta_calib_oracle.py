"""CPU oracle for offline per-head threshold calibration: frozen constants c_h
that replace the threshold projection for a stationary deployment.

TEST INFRASTRUCTURE ONLY.  Only the test suite may import or run this module.
It shares no code with the CUDA library and does not import it.

Source: "Elastic Threshold Attention: Learned Contextual Sparsity for
Long-Context Decoding", section 4.7 (distilling static thresholds: a
1/t-weighted score histogram over calibration sequences, then a binary search
for each head's target density) and Appendix D.2 (its algorithm; the body of
that appendix is lost from the pages).  Reading used here: every causal
(query t, key j <= t) logit S_tj = scale q_t . k_j of a head enters with
weight 1/(t + 1), so each query row carries total weight 1 whatever its
length; the density at a constant c is the weighted fraction of logits with
S_tj >= c, i.e. the mean over rows of the fraction of keys at or above c; the
constant of a head is the c at which that density equals the head's target.

Two solvers: ``exact_constant`` sorts the weighted logits (the definition);
``histogram_constant`` works from a binned histogram as a deployment would,
searching the bins from the top and interpolating linearly inside the bin
that crosses the target (its error is at most one bin width).

Parity status: pinned by tests/test_oracle_calib_pins.py (brute-force loops,
the total weight B T, closed forms on constructed logits, monotonicity, the
histogram solver within one bin of the exact one).
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        return x.detach().float().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def head_logits(q_rows, K, scale: float):
    """All causal logits of one head and sequence with their weights:
    (S [n], w [n]) over the pairs (t, j <= t), t < T = len(q_rows)."""
    q, k = _f64(q_rows), _f64(K)
    T = q.shape[0]
    S = scale * (q @ k[:T].T)
    tri = np.tril(np.ones((T, T), dtype=bool))
    w = np.broadcast_to((1.0 / (np.arange(T) + 1.0))[:, None], (T, T))
    return S[tri], w[tri]


def calibration_logits(q, k, seq_len: int, scale: Optional[float] = None) -> Dict[int, tuple]:
    """Per query head h: (S, w) over every sequence of the batch.  q [B, Hq, T, d],
    k [B, Hkv, >= T, d]; head h reads KV head h // G."""
    q, k = _f64(q), _f64(k)
    B, Hq, T, d = q.shape
    G = Hq // k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    res = {}
    for h in range(Hq):
        Ss, ws = [], []
        for b in range(B):
            S, w = head_logits(q[b, h, :seq_len], k[b, h // G, :seq_len], scale)
            Ss.append(S)
            ws.append(w)
        res[h] = (np.concatenate(Ss), np.concatenate(ws))
    return res


def histogram(S, w, lo: float, hi: float, nbins: int) -> np.ndarray:
    """Weighted histogram with nbins equal bins over [lo, hi) plus an
    underflow slot (index 0) and an overflow slot (index nbins + 1)."""
    width = (hi - lo) / nbins
    idx = np.floor((np.asarray(S) - lo) / width).astype(np.int64)
    idx = np.clip(idx, -1, nbins) + 1
    out = np.zeros(nbins + 2)
    np.add.at(out, idx, np.asarray(w))
    return out


def density(S, w, c: float) -> float:
    """Weighted fraction of logits at or above c."""
    S, w = np.asarray(S), np.asarray(w)
    return float(w[S >= c].sum() / w.sum())


def exact_constant(S, w, target: float) -> float:
    """Largest c with density(c) >= target (a logit value)."""
    order = np.argsort(-np.asarray(S), kind="stable")
    Ss = np.asarray(S)[order]
    cw = np.cumsum(np.asarray(w)[order]) / np.sum(w)
    k = int(np.searchsorted(cw, target - 1e-15))
    return float(Ss[min(k, len(Ss) - 1)])


def histogram_constant(hist, lo: float, hi: float, target: float) -> float:
    """The constant from a histogram: walk down from the top bin until the
    weight above reaches target of the total; interpolate inside that bin."""
    hist = np.asarray(hist, dtype=np.float64)
    nbins = len(hist) - 2
    width = (hi - lo) / nbins
    total = hist.sum()
    need = target * total
    acc = hist[nbins + 1]
    if acc >= need:
        return hi
    for b in range(nbins, 0, -1):  # slot b holds [lo + (b-1) w, lo + b w)
        if acc + hist[b] >= need:
            frac = (need - acc) / hist[b]
            return lo + b * width - frac * width
        acc += hist[b]
    return lo
