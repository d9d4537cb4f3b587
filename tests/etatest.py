"""Helpers shared by the GPU parity tests: run a workload through the CUDA
library (C ABI via the binding) and compare it with the CPU oracle.

Comparison rules (written out here so every test uses the same ones):
  * admitted block sets, per query head and per GQA union, must be identical;
    the one allowance is a block whose oracle margin |Score - tau~| is below
    the fp32 rounding band SCREEN_EPS: the device decides the bound in fp32
    (Appendix F.2 of the ETA pages), so either decision is correct there.  For
    such a head the oracle's output is taken for the admitted set the device
    chose, which must differ from the oracle's own set only on those blocks.
  * outputs within OUT_TOL[dtype] max-abs, lse within LSE_TOL[dtype].
"""
from __future__ import annotations

import math

import numpy as np
import torch

import learned_threshold_sparse_b200 as eta
import oracle

SCREEN_EPS = 2e-4
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


def compare(wl, g, r, out_tol=None, lse_tol=None, screen_eps=SCREEN_EPS, heads=None):
    """Assert device results g equal oracle results r under the rules above.
    Returns the number of (head, block) decisions that fell in the band."""
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
            margin = r["scores"][i, h, :nb] - r["tau_tilde"][i, h]
            band = np.abs(np.nan_to_num(margin, nan=np.inf)) < screen_eps
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
