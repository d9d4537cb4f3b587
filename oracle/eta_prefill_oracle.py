"""CPU oracle for the causal ETA forward pass over a whole sequence (the
training forward / prefill step).

TEST INFRASTRUCTURE ONLY.  Only the test suite and the benchmark's CPU-baseline
leg may import or run this module.  It shares no code with the CUDA library and
does not import it.

Follows "Elastic Threshold Attention: Learned Contextual Sparsity for
Long-Context Decoding":

* section 2.3 (efficient fused training kernel) and Appendix E.1 (forward
  pass formulation): queries are processed with their own predicted
  thresholds tau_i, keys causally (key j is seen by query i iff j <= i);
* Appendix E.3: the inclusion probability sigma_ij = sigmoid(beta (S_ij -
  tau_i)) enters twice, as the multiplicative mask S~_ij = S_ij sigma_ij of
  the softmax logits and as the row sum R_i = sum_j sigma_ij that feeds the
  sparsity regulariser;
* Appendix E.4 (space bullet): the forward pass keeps O, the log-sum-exp L and
  the row vector Sigma (read here as R) for the backward pass.

The threshold per query row is the decode step's: tau_i = w_tau . q_i + b_tau
(learned) or the frozen per-head constant c, minus the offset a (section 1;
Appendix D; Appendix G.1).  Everything is float64 from the exact bf16/fp32
inputs.

Parity status: pinned by tests/test_oracle_prefill_pins.py (library causal
attention at sigma = 1 and at beta = 0, closed forms of the first row and of R,
a brute-force loop, agreement of the last row with the decode oracle).
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (bf16 is widened exactly)
        return x.detach().float().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def prefill_thresholds(q_rows, tau_mode: str, w_h=None, b_h=None, c_h=None, offset_a: float = 0.0) -> np.ndarray:
    """tau~_i for every query row of one head: w . q_i + b - a (learned) or
    c - a (calibrated)."""
    q_rows = _f64(q_rows)
    if tau_mode == "learned":
        return q_rows @ _f64(w_h) + float(b_h) - offset_a
    if tau_mode == "calibrated":
        return np.full(q_rows.shape[0], float(c_h) - offset_a)
    raise ValueError(tau_mode)


def prefill_head(q, K, V, tau_tilde, scale: float, beta: float):
    """Causal tempered attention of one head over T query rows.

    S_ij = scale q_i . k_j for j <= i; sigma_ij = sigmoid(beta (S_ij - tau_i));
    S~_ij = S_ij sigma_ij; o_i = sum_j e^{S~_ij} v_j / sum_j e^{S~_ij};
    L_i = ln sum_j e^{S~_ij}; R_i = sum_j sigma_ij.  Returns (O [T, d], L [T],
    R [T])."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    tau = _f64(tau_tilde)
    T = q.shape[0]
    S = scale * (q @ K[:T].T)
    causal = np.tril(np.ones((T, T), dtype=bool))
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-beta * (S - tau[:, None])))
    sig = np.where(causal, sig, 0.0)
    St = np.where(causal, S * sig, -np.inf)
    m = St.max(axis=1)
    w = np.exp(St - m[:, None])
    l = w.sum(axis=1)
    O = (w @ V[:T]) / l[:, None]
    return O, m + np.log(l), sig.sum(axis=1)


def prefill_row(q_i, K_seen, V_seen, tau_i: float, scale: float, beta: float):
    """One query row of the causal pass: row i sees the keys K_seen = k_0..k_i
    (all of them, no mask).  Same quantities as prefill_head for that row:
    (o_i [d], L_i, R_i).  Lets a test check sampled rows of a long sequence
    without the T x T matrix."""
    q_i, K, V = _f64(q_i), _f64(K_seen), _f64(V_seen)
    S = scale * (K @ q_i)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-beta * (S - float(tau_i))))
    St = S * sig
    m = St.max()
    w = np.exp(St - m)
    l = w.sum()
    return (w @ V) / l, m + np.log(l), sig.sum()


def prefill(q, k, v, seq_len: int, tau_mode: str, w_tau=None, b_tau=None, c_tau=None,
            scale: Optional[float] = None, beta: float = 5.0, offset_a: float = 0.0) -> Dict[str, np.ndarray]:
    """Whole batch: q [B, Hq, T, d], k and v [B, Hkv, >= T, d]; query head h
    reads KV head h // G (contiguous GQA grouping).  Returns out [B, Hq, T, d],
    lse [B, Hq, T] and gate_sum [B, Hq, T]."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, T, d = q.shape
    assert T == seq_len
    Hkv = k.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Hq, T, d))
    lse = np.zeros((B, Hq, T))
    gate = np.zeros((B, Hq, T))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            tau = prefill_thresholds(q[b, h], tau_mode,
                                     None if w_tau is None else _f64(w_tau)[h],
                                     None if b_tau is None else _f64(b_tau)[h],
                                     None if c_tau is None else _f64(c_tau)[h], offset_a)
            O, L, R = prefill_head(q[b, h], k[b, g, :T], v[b, g, :T], tau, scale, beta)
            out[b, h], lse[b, h], gate[b, h] = O, L, R
    return {"out": out, "lse": lse, "gate_sum": gate}


def prefill_flops(batch: int, n_q_heads: int, seq_len: int, head_dim: int) -> float:
    """Tensor flops of the two contractions (S = Q K^T and O = P V) over the
    causal triangle: 2 x 2 d per (query, key) pair with key <= query."""
    pairs = seq_len * (seq_len + 1) / 2
    return 4.0 * head_dim * pairs * batch * n_q_heads
