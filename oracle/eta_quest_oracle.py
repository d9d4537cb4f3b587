"""CPU oracle for the coordinate-box block bound the pages compare against
(Quest), and for the token-recall study of the two screens.

TEST INFRASTRUCTURE ONLY.  Only the test suite (and the recall study script
beside this file) may import or run this module.  It shares no code with the
CUDA library and does not import it.

Source: "Elastic Threshold Attention: Learned Contextual Sparsity for
Long-Context Decoding", section 4.3, "Comparison with Quest": Quest bounds a
block by summing per-coordinate extrema,
    sum_i max(q_i kmax_i, q_i kmin_i),
and the pages report that ETA's dual bound captures a higher fraction of the
true above-threshold keys (token recall, Table 3; geometric analysis in
Appendix K).  Readings used here: the per-coordinate extrema are stored in
fp16 rounded outward (minimum toward -inf, maximum toward +inf), so the box
bound stays a strict upper bound of every key's logit; a key is "true" when
scale q . k >= tau~; token recall of an admitted block set is the fraction of
true keys that lie in admitted blocks; the two screens are compared at the
dual screen's own threshold and at matched density (the same number of
blocks per head, taken in descending order of each bound).

Parity status: pinned by tests/test_oracle_quest_pins.py (strictness by brute
force, closed forms for sign-constant queries and one-key blocks, outward
rounding against the exact extrema, recall of a constructed case).
"""
from __future__ import annotations

from typing import Dict, Sequence

import numpy as np

import oracle


def _f16_down(x):
    """Largest fp16 value <= x."""
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    over = h.astype(np.float64) > x
    return np.where(over, np.nextafter(h, np.float16(-np.inf)), h).astype(np.float16)


def _f16_up(x):
    """Smallest fp16 value >= x."""
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    under = h.astype(np.float64) < x
    return np.where(under, np.nextafter(h, np.float16(np.inf)), h).astype(np.float16)


def box_summary(k_block):
    """(kmin, kmax) fp16 of one block [n, d], rounded outward."""
    k = oracle.as_f64(k_block)
    return _f16_down(k.min(axis=0)), _f16_up(k.max(axis=0))


def summarize_box(k, seq_lens: Sequence[int], b: int) -> Dict[str, np.ndarray]:
    """Box metadata of a cache k [B, Hkv, max_ctx, d]: kmin, kmax
    [B, Hkv, nbmax, d] fp16 (zero past each sequence's last block)."""
    B, Hkv, Tmax, d = k.shape
    nbmax = (Tmax + b - 1) // b
    lo = np.zeros((B, Hkv, nbmax, d), np.float16)
    hi = np.zeros((B, Hkv, nbmax, d), np.float16)
    for i, T in enumerate(seq_lens):
        for g in range(Hkv):
            for j in range((T + b - 1) // b):
                lo[i, g, j], hi[i, g, j] = box_summary(k[i, g, j * b:min(T, (j + 1) * b)])
    return {"kmin": lo, "kmax": hi}


def box_scores(q, kmin, kmax, scale: float) -> np.ndarray:
    """scale sum_i max(q_i kmin_i, q_i kmax_i) per block: [nb]."""
    q = oracle.as_f64(q)
    a = q * kmin.astype(np.float64)
    c = q * kmax.astype(np.float64)
    return scale * np.maximum(a, c).sum(axis=-1)


def token_recall(q, K, T: int, b: int, tau_tilde: float, scale: float, admitted: np.ndarray):
    """(true keys, recalled true keys) of one head: keys s < T with
    scale q . k_s >= tau~, and those of them inside admitted blocks."""
    S = scale * (oracle.as_f64(K)[:T] @ oracle.as_f64(q))
    true = S >= tau_tilde
    inblk = np.repeat(np.asarray(admitted, bool), b)[:T]
    return int(true.sum()), int((true & inblk).sum())


def recall_study(wl, n_local_blocks: int = 2) -> Dict[str, float]:
    """Token recall and block density of the dual screen and of the box screen
    over every (sequence, query head) of a workload: at tau~ (each bound used
    as a screen, with the always-loaded window) and at matched density (the
    box screen keeps as many blocks as the dual screen admitted)."""
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, wl.block_size, wl.tau_mode, w_tau=wl.w_tau,
                      b_tau=wl.b_tau, c_tau=wl.c_tau, scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a,
                      z=wl.z, n_local_blocks=n_local_blocks, heads=[])
    box = summarize_box(wl.k, wl.seq_lens, wl.block_size)
    G = wl.n_q_heads // wl.n_kv_heads
    tot = dict(true=0, dual=0, box_tau=0, box_matched=0, blocks=0, dual_blocks=0, box_tau_blocks=0)
    for i, T in enumerate(wl.seq_lens):
        nb = (T + wl.block_size - 1) // wl.block_size
        if nb == 0:
            continue
        for h in range(wl.n_q_heads):
            g = h // G
            tt = r["tau_tilde"][i, h]
            q = wl.q[i, h]
            K = wl.k[i, g]
            adm_dual = r["admitted"][i, h, :nb]
            sc = box_scores(q, box["kmin"][i, g, :nb], box["kmax"][i, g, :nb], wl.scale)
            adm_box, _ = oracle.admit(sc, tt, nb, n_local_blocks, True)
            n = int(adm_dual.sum())
            top = np.zeros(nb, bool)
            top[np.argsort(-sc, kind="stable")[:n]] = True
            t_all, t_dual = token_recall(q, K, T, wl.block_size, tt, wl.scale, adm_dual)
            _, t_box = token_recall(q, K, T, wl.block_size, tt, wl.scale, adm_box)
            _, t_top = token_recall(q, K, T, wl.block_size, tt, wl.scale, top)
            tot["true"] += t_all
            tot["dual"] += t_dual
            tot["box_tau"] += t_box
            tot["box_matched"] += t_top
            tot["blocks"] += nb
            tot["dual_blocks"] += n
            tot["box_tau_blocks"] += int(adm_box.sum())
    den = max(tot["true"], 1)
    return {
        "true_keys": tot["true"],
        "recall_dual": tot["dual"] / den,
        "recall_box_at_tau": tot["box_tau"] / den,
        "recall_box_matched_density": tot["box_matched"] / den,
        "density_dual": tot["dual_blocks"] / tot["blocks"],
        "density_box_at_tau": tot["box_tau_blocks"] / tot["blocks"],
    }
