"""CPU oracle for the Elastic Threshold Attention (ETA) single-token decode step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
the CPU-baseline leg of the benchmark may import or run this module.  It shares
no code with the CUDA library and does not import it.

Every value is computed in float64 from the exact fp32/bf16 inputs, unless the
method fixes a storage precision (the fp16 block centroid and spread and the
fp32 block norm of Appendix F.1).  The functions follow the pages of
"Elastic Threshold Attention: Learned Contextual Sparsity for Long-Context
Decoding" in their own order:

* threshold:      tau = w_tau . q + b_tau, or a frozen per-head constant c
                  (section 1; Appendix D.1; section 4.7 / D.2), and the
                  effective threshold tau~ = tau - a (Appendix G.1).
* block summary:  centroid mu_B, coordinate standard deviation sigma_B (fp16)
                  and scalar maximum norm M_B (fp32) per block per KV head
                  (Appendix F.1; section 3.2).
* block screen:   an O(1) bound per (head, block) from (mu_B, sigma_B, M_B)
                  compared with tau~ (section 3.1; section 4.3 "Dual Bound";
                  Appendix F.1 step 1).  The printed form of the bound is lost
                  from the pages; the reading used here is documented in
                  ``block_scores``.
* admission:      GQA union loading (Appendix F.1 step 2), the always-loaded
                  recent window lwb = 2 plus the tail block (section 4.8),
                  top-1 rescue (Appendix F.4).
* attention:      S = q k / sqrt(d_k), S~ = S * sigmoid(beta (S - tau~)),
                  w = exp(S~), o = sum w v / sum w (section 2.2; Appendix G.1;
                  Appendix E.3 "Multiplicative Masking").
* split merge:    associative online-softmax merge of chunk partials
                  (section 3.2; Appendix F.3).

Parity status: every function here is pinned by the tests in
``tests/test_oracle_pins.py`` except the exact algebraic form of the dual bound
(the equation is missing from the pages): its two halves are pinned separately
(the geometric half as a true upper bound by brute force, the probabilistic half
by closed forms), the combination by ``min`` is a reading and is
"parity unpinned" against the pages.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

LOG2E = 1.0 / math.log(2.0)


# ------------------------------------------------------------------ rounding

def fp16_round(x) -> np.ndarray:
    """Round to IEEE binary16, nearest-even (storage precision of mu_B and
    sigma_B, Appendix F.1)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


def fp32_round_up(x) -> np.ndarray:
    """Smallest fp32 value >= x (storage precision of M_B, Appendix F.1; rounding
    up keeps M_B an upper bound of the exact norm)."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    low = f.astype(np.float64) < x
    return np.where(low, np.nextafter(f, np.float32(np.inf)), f).astype(np.float32)


def as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (bf16 or fp32): exact widening
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


# ------------------------------------------------------------- block summary

def block_summary(k_block) -> Tuple[np.ndarray, np.ndarray, np.float32]:
    """Summary of one KV block: (mu_hat fp16 [d], sigma_hat fp16 [d], M fp32).

    mu = mean of the block's keys; sigma = population standard deviation per
    coordinate (the pages store sigma rather than sigma^2 to avoid fp16
    underflow, Appendix F.1); M = max over the block's keys of ||k_s - mu_hat||,
    measured from the stored (fp16) centroid and rounded up to fp32.
    """
    k = as_f64(k_block)
    n = k.shape[0]
    mu = k.sum(axis=0) / n
    sigma = np.sqrt(((k - mu) ** 2).sum(axis=0) / n)
    mu_hat = fp16_round(mu)
    dev = k - mu_hat.astype(np.float64)
    m = np.sqrt((dev * dev).sum(axis=1)).max()
    return mu_hat, fp16_round(sigma), fp32_round_up(m)


def sequence_summary(k_seq, T: int, b: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Summaries of every block of one (sequence, KV head): blocks cover tokens
    [j b, min((j+1) b, T)).  Returns mu_hat [nb, d] fp16, sigma_hat [nb, d] fp16,
    M [nb] fp32."""
    k = as_f64(k_seq)[:T]
    d = k.shape[1]
    nb = (T + b - 1) // b
    mu = np.zeros((nb, d), np.float16)
    sg = np.zeros((nb, d), np.float16)
    mm = np.zeros((nb,), np.float32)
    nfull = T // b
    if nfull:
        kb = k[: nfull * b].reshape(nfull, b, d)
        mean = kb.sum(axis=1) / b
        std = np.sqrt(((kb - mean[:, None, :]) ** 2).sum(axis=1) / b)
        mu[:nfull] = fp16_round(mean)
        sg[:nfull] = fp16_round(std)
        dev = kb - mu[:nfull].astype(np.float64)[:, None, :]
        mm[:nfull] = fp32_round_up(np.sqrt((dev * dev).sum(axis=2)).max(axis=1))
    if nb > nfull:
        mu[nfull], sg[nfull], mm[nfull] = block_summary(k[nfull * b:T])
    return mu, sg, mm


# ----------------------------------------------------------------- threshold

def threshold_learned(q, w_tau, b_tau, offset_a: float) -> float:
    """tau~ = (w_tau . q + b_tau) - a: query-conditioned threshold of one head
    (section 1; Appendix D.1) minus the offset a (Appendix G.1)."""
    return float(as_f64(w_tau) @ as_f64(q) + float(b_tau)) - float(offset_a)


def threshold_calibrated(c_tau, offset_a: float) -> float:
    """tau~ = c - a with a frozen per-head constant c (section 4.7; D.2)."""
    return float(c_tau) - float(offset_a)


# ------------------------------------------------------------------- screen

def block_scores(q, mu_hat, sigma_hat, max_norm, scale: float, z: float) -> np.ndarray:
    """Per-block upper estimate of the largest scaled logit in the block.

    Reading of the lost "Dual Bound" (section 4.3, Equation 7; Appendix F.1):
      geometric half      <q, mu> + ||q|| M           (Cauchy-Schwarz on the
                          ball of radius M around the stored centroid: a strict
                          upper bound of every key's logit in the block)
      probabilistic half  <q, mu> + z sqrt(sum_i q_i^2 sigma_i^2)
                          (z standard deviations of q.k under the block's
                          per-coordinate spread)
      Score = scale * (<q, mu> + min(||q|| M, z ||sigma (.) q||)).
    z = +inf leaves only the geometric half (strict screening).
    """
    q = as_f64(q)
    mu = np.asarray(mu_hat, dtype=np.float64)
    sg = np.asarray(sigma_hat, dtype=np.float64)
    m = np.asarray(max_norm, dtype=np.float64)
    centre = mu @ q
    geometric = np.sqrt(q @ q) * m
    if math.isinf(z):
        spread = geometric
    else:
        prob = z * np.sqrt((sg * sg) @ (q * q))
        spread = np.minimum(geometric, prob)
    return scale * (centre + spread)


def screened_and_forced(nb: int, n_local_blocks: int) -> Tuple[np.ndarray, np.ndarray]:
    """Which blocks are screened and which are always loaded.

    With n_local_blocks = lwb >= 0 the block holding the newest token plus the
    lwb blocks before it are always loaded (section 4.8: "lwb = 2 plus the tail
    block"); the partial tail block is therefore never screened (Appendix F.4).
    lwb = -1 disables the always-loaded window: every block, the tail included,
    is screened."""
    j = np.arange(nb)
    if n_local_blocks < 0:
        return np.ones(nb, bool), np.zeros(nb, bool)
    first_forced = max(0, nb - 1 - n_local_blocks)
    return j < first_forced, j >= first_forced


def admit(scores: np.ndarray, tau_tilde: float, nb: int, n_local_blocks: int,
          screen_enabled: bool = True) -> Tuple[np.ndarray, bool]:
    """Admitted block set of one query head.

    A screened block is admitted iff Score >= tau~ (section 3.1 "significant":
    S >= tau; section 2.2 salient set uses S >= tau~).  Always-loaded blocks are
    added.  If nothing is admitted, the single block with the highest Score is
    admitted (top-1 rescue, Appendix F.4), lowest index on ties.  With the
    screen disabled every block is admitted.
    Returns (admitted [nb] bool, rescue_fired)."""
    if not screen_enabled:
        return np.ones(nb, bool), False
    screened, forced = screened_and_forced(nb, n_local_blocks)
    adm = forced.copy()
    adm[screened] |= scores[screened] >= tau_tilde
    if nb > 0 and not adm.any():
        cand = np.where(screened, scores, -np.inf)
        adm[int(np.argmax(cand))] = True
        return adm, True
    return adm, False


# ----------------------------------------------------------------- attention

def sigmoid(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def tempered_logits(S, tau_tilde: float, beta: float) -> np.ndarray:
    """Centred-SiLU tempering S~ = S * sigmoid(beta (S - tau~)) (section 2.2;
    Appendix E.3 multiplicative masking; Appendix G.1)."""
    S = np.asarray(S, dtype=np.float64)
    return S * sigmoid(beta * (S - tau_tilde))


def token_mask(admitted: np.ndarray, T: int, b: int) -> np.ndarray:
    """Tokens of the admitted blocks that exist (position < T)."""
    return np.repeat(admitted, b)[:T]


def partial_state(q, K, V, tau_tilde: float, scale: float, beta: float,
                  mask: np.ndarray) -> Tuple[np.ndarray, float, float]:
    """Unnormalised partial of one token subset: (sum_s e^{S~_s - m} v_s, m, l)
    with m = max S~ and l = sum e^{S~_s - m}; an empty subset gives
    (0, -inf, 0)."""
    q = as_f64(q)
    Kx = as_f64(K)[mask]
    Vx = as_f64(V)[mask]
    d = q.shape[0]
    if Kx.shape[0] == 0:
        return np.zeros(d), -math.inf, 0.0
    St = tempered_logits(scale * (Kx @ q), tau_tilde, beta)
    m = float(St.max())
    w = np.exp(St - m)
    return w @ Vx, m, float(w.sum())


def combine_partials(parts: Sequence[Tuple[np.ndarray, float, float]]) -> Tuple[np.ndarray, float]:
    """Associative merge of split partials (section 3.2; Appendix F.3):
    m* = max m_c, l* = sum l_c e^{m_c - m*}, o = sum e^{m_c - m*} acc_c / l*,
    lse = m* + ln l*.  All-empty input gives (0, -inf)."""
    ms = [p[1] for p in parts if p[2] > 0]
    d = parts[0][0].shape[0]
    if not ms:
        return np.zeros(d), -math.inf
    mstar = max(ms)
    acc = np.zeros(d)
    l = 0.0
    for a, m, lc in parts:
        if lc <= 0:
            continue
        f = math.exp(m - mstar)
        acc += f * a
        l += f * lc
    return acc / l, mstar + math.log(l)


def attend_head(q, K, V, T: int, b: int, admitted: np.ndarray, tau_tilde: float,
                scale: float, beta: float) -> Tuple[np.ndarray, float]:
    """Tempered attention of one query head over the tokens of its admitted
    blocks (section 2.2: o = Z^-1 sum w_s v_s with w_s = exp(S~_s)).
    Returns (o [d], lse)."""
    mask = token_mask(admitted, T, b)
    return combine_partials([partial_state(q, K[:T], V[:T], tau_tilde, scale, beta, mask)])


def attend_head_chunked(q, K, V, T: int, b: int, admitted: np.ndarray, tau_tilde: float,
                        scale: float, beta: float, chunk_blocks: int) -> Tuple[np.ndarray, float]:
    """Same result computed as split-KV chunks of ``chunk_blocks`` admitted
    blocks each, merged with ``combine_partials`` (section 3.2; Appendix F.3)."""
    ids = np.flatnonzero(admitted)
    parts = []
    for c in range(0, max(len(ids), 1), chunk_blocks):
        sub = np.zeros_like(admitted)
        sub[ids[c:c + chunk_blocks]] = True
        parts.append(partial_state(q, K[:T], V[:T], tau_tilde, scale, beta, token_mask(sub, T, b)))
    return combine_partials(parts)


# -------------------------------------------------------------- whole step

def summarize(k, seq_lens: Sequence[int], b: int) -> Dict[str, np.ndarray]:
    """Oracle metadata for a whole cache k [B, Hkv, max_ctx, d]:
    mu [B, Hkv, nbmax, d] fp16, sigma same, M [B, Hkv, nbmax] fp32 (zero past
    each sequence's last block)."""
    B, Hkv, Tmax, d = k.shape
    nbmax = (Tmax + b - 1) // b
    mu = np.zeros((B, Hkv, nbmax, d), np.float16)
    sg = np.zeros((B, Hkv, nbmax, d), np.float16)
    mm = np.zeros((B, Hkv, nbmax), np.float32)
    for i, T in enumerate(seq_lens):
        nb = (T + b - 1) // b
        for g in range(Hkv):
            if nb:
                mu[i, g, :nb], sg[i, g, :nb], mm[i, g, :nb] = sequence_summary(k[i, g], T, b)
    return {"mu": mu, "sigma": sg, "max_norm": mm}


def decode(q, k, v, seq_lens: Sequence[int], block_size: int, tau_mode: str,
           w_tau=None, b_tau=None, c_tau=None, scale: float = None, beta: float = 5.0,
           offset_a: float = 0.0, z: float = 2.0, n_local_blocks: int = 2,
           screen_enabled: bool = True, summary: Optional[Dict[str, np.ndarray]] = None,
           heads: Optional[Sequence[Tuple[int, int]]] = None) -> Dict[str, np.ndarray]:
    """The whole decode step for every (sequence, query head).

    q [B, Hq, d]; k, v [B, Hkv, max_ctx, d]; query head h reads KV head
    h // (Hq / Hkv) (contiguous GQA grouping).  ``heads`` restricts the
    attention outputs to the listed (sequence, head) pairs (the screen is
    always computed for every head).  Returns a dict of arrays:
      o [B, Hq, d], lse [B, Hq], tau_tilde [B, Hq],
      scores [B, Hq, nbmax] (NaN where a block is not screened),
      admitted [B, Hq, nbmax] bool, rescued [B, Hq] bool,
      union [B, Hkv, nbmax] bool, union_mask [B, Hkv, nbmax] uint32,
      admitted_count [B, Hq], union_count [B, Hkv], and the metadata used.
    """
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    b = block_size
    nbmax = (k.shape[2] + b - 1) // b
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if summary is None:
        summary = summarize(k, seq_lens, b)
    qf = as_f64(q)
    out = {
        "o": np.zeros((B, Hq, d)),
        "lse": np.full((B, Hq), -math.inf),
        "tau_tilde": np.zeros((B, Hq)),
        "scores": np.full((B, Hq, nbmax), np.nan),
        "admitted": np.zeros((B, Hq, nbmax), bool),
        "rescued": np.zeros((B, Hq), bool),
        "union": np.zeros((B, Hkv, nbmax), bool),
        "union_mask": np.zeros((B, Hkv, nbmax), np.uint32),
    }
    want = set(heads) if heads is not None else None
    for i, T in enumerate(seq_lens):
        nb = (T + b - 1) // b
        for g in range(Hkv):
            Kf = as_f64(k[i, g, :T])
            Vf = as_f64(v[i, g, :T])
            mu = summary["mu"][i, g, :nb]
            sg = summary["sigma"][i, g, :nb]
            mm = summary["max_norm"][i, g, :nb]
            for j in range(G):
                h = g * G + j
                if tau_mode == "learned":
                    tt = threshold_learned(qf[i, h], w_tau[h], b_tau[h], offset_a)
                else:
                    tt = threshold_calibrated(c_tau[h], offset_a)
                out["tau_tilde"][i, h] = tt
                sc = block_scores(qf[i, h], mu, sg, mm, scale, z) if nb else np.zeros(0)
                screened, _ = screened_and_forced(nb, n_local_blocks)
                out["scores"][i, h, :nb] = np.where(screened, sc, np.nan) if screen_enabled else np.nan
                adm, resc = admit(sc, tt, nb, n_local_blocks, screen_enabled)
                out["admitted"][i, h, :nb] = adm
                out["rescued"][i, h] = resc
                out["union"][i, g, :nb] |= adm
                out["union_mask"][i, g, :nb] |= (adm.astype(np.uint32) << j)
                if want is not None and (i, h) not in want:
                    continue
                if T > 0:
                    o, lse = attend_head(qf[i, h], Kf, Vf, T, b, adm, tt, scale, beta)
                    out["o"][i, h], out["lse"][i, h] = o, lse
    out["admitted_count"] = out["admitted"].sum(axis=2)
    out["union_count"] = out["union"].sum(axis=2)
    out.update(summary)
    return out


def densities(result: Dict[str, np.ndarray], seq_lens: Sequence[int], b: int) -> Dict[str, np.ndarray]:
    """Per-head density |A_h| / nb, GQA-union density |U_g| / nb and the
    attended-token fraction (the integer selection counts of Appendix F.4,
    divided by the number of blocks / tokens)."""
    B, Hq = result["admitted_count"].shape
    Hkv = result["union_count"].shape[1]
    head = np.zeros((B, Hq))
    union = np.zeros((B, Hkv))
    tok = np.zeros((B, Hq))
    for i, T in enumerate(seq_lens):
        nb = (T + b - 1) // b
        if nb == 0:
            continue
        head[i] = result["admitted_count"][i] / nb
        union[i] = result["union_count"][i] / nb
        sizes = np.minimum(b, T - np.arange(nb) * b)
        tok[i] = (result["admitted"][i, :, :nb] * sizes[None, :]).sum(axis=1) / T
    return {"head": head, "union": union, "token_fraction": tok}


def metadata_record_bytes(head_dim: int) -> int:
    """Bytes of one per-block, per-KV-head record: fp16 centroid [d], fp16
    standard deviation [d], fp32 maximum norm (Appendix F.1)."""
    return 2 * head_dim + 2 * head_dim + 4
