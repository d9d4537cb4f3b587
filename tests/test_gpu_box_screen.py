"""The comparison coordinate-box (Quest) screen on the device against the box
oracle: per-coordinate fp16 extrema rounded outward bit-exact, and decode
steps screened with the box bound under the same comparison rules as the
dual bound (identical admitted sets up to decisions inside the fp32 error
bound, outputs within tolerance)."""
import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import oracle
import workloads
from etatest import compare, gpu_decode, upload
from oracle import eta_quest_oracle as qo

pytestmark = pytest.mark.gpu

F32, BF16 = workloads.F32, workloads.BF16


def _box_summary(wl, t):
    s = eta.alloc_summary(wl.batch, wl.n_kv_heads, wl.max_ctx, wl.head_dim, wl.block_size, fmt="box")
    first = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    eta.eta_block_summary_update(t["k"], t["v"], t["seq"], s, wl.block_size, first, wl.nb_max, wl.n_q_heads)
    torch.cuda.synchronize()
    return s


def _oracle_box_decode(wl):
    """The oracle decode with the box bound as the screen: thresholds from the
    decode oracle, admission by oracle.admit over the box scores, attention by
    oracle.attend_head over that set."""
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, wl.block_size, wl.tau_mode, w_tau=wl.w_tau, b_tau=wl.b_tau,
                      c_tau=wl.c_tau, scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
                      n_local_blocks=wl.n_local_blocks, heads=[])
    box = qo.summarize_box(wl.k, wl.seq_lens, wl.block_size)
    G = wl.n_q_heads // wl.n_kv_heads
    r["admitted"][:] = False
    r["union"][:] = False
    for i, T in enumerate(wl.seq_lens):
        nb = wl.n_blocks(i)
        for h in range(wl.n_q_heads):
            g = h // G
            tt = r["tau_tilde"][i, h]
            sc = qo.box_scores(wl.q[i, h], box["kmin"][i, g, :nb], box["kmax"][i, g, :nb], wl.scale)
            screened, _ = oracle.screened_and_forced(nb, wl.n_local_blocks)
            r["scores"][i, h, :nb] = np.where(screened, sc, np.nan)
            adm, _ = oracle.admit(sc, tt, nb, wl.n_local_blocks, True)
            r["admitted"][i, h, :nb] = adm
            r["union"][i, g, :nb] |= adm
            if T > 0:
                r["o"][i, h], r["lse"][i, h] = oracle.attend_head(oracle.as_f64(wl.q[i, h]),
                                                                  oracle.as_f64(wl.k[i, g, :T]),
                                                                  oracle.as_f64(wl.v[i, g, :T]), T,
                                                                  wl.block_size, adm, tt, wl.scale, wl.beta)
    r["admitted_count"] = r["admitted"].sum(axis=2)
    r["union_count"] = r["union"].sum(axis=2)
    r["kmin"], r["kmax"] = box["kmin"], box["kmax"]  # the metadata this screen read
    return r


@pytest.mark.parametrize("case", [
    dict(dtype=BF16, d=128, b=64, lens=[1000, 1, 64, 0], kind="cluster"),
    dict(dtype=F32, d=64, b=32, lens=[777]),
])
def test_box_extrema_bit_exact(case):
    wl = workloads.custom(seed=51, batch=len(case["lens"]), n_q_heads=4, n_kv_heads=2, head_dim=case["d"],
                          block_size=case["b"], seq_lens=case["lens"], dtype=case["dtype"],
                          key_kind=case.get("kind", "normal"))
    t = upload(wl)
    s = _box_summary(wl, t)
    ref = qo.summarize_box(wl.k, wl.seq_lens, wl.block_size)
    for i in range(wl.batch):
        nb = wl.n_blocks(i)
        np.testing.assert_array_equal(s["mu"][i, :, :nb].cpu().numpy(), ref["kmin"][i, :, :nb])
        np.testing.assert_array_equal(s["sigma"][i, :, :nb].cpu().numpy(), ref["kmax"][i, :, :nb])


BOX_DECODE = [
    dict(id="g4_bf16_cluster_ragged", seed=2, B=4, Hq=16, Hkv=4, d=128, b=64, lens=[3000, 1, 64, 777],
         dtype=BF16, mode="calibrated", kind="cluster", bias=1.0),
    dict(id="g8_bf16_d64_b32_cluster", seed=3, B=1, Hq=16, Hkv=2, d=64, b=32, lens=[2500], dtype=BF16,
         kind="cluster", bias=2.0, std=1.0),
    dict(id="g1_f32_d64_b64", seed=1, B=1, Hq=4, Hkv=4, d=64, b=64, lens=[1000], dtype=F32, bias=6.0, std=1.0),
]


@pytest.mark.parametrize("c", BOX_DECODE, ids=[c["id"] for c in BOX_DECODE])
def test_box_screen_decode_parity(c):
    wl = workloads.custom(seed=c["seed"], batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                          head_dim=c["d"], block_size=c["b"], seq_lens=c["lens"], dtype=c["dtype"],
                          tau_mode=c.get("mode", "learned"), key_kind=c.get("kind", "normal"),
                          tau_bias=c["bias"], tau_std=c.get("std", 0.0))
    t = upload(wl)
    g = gpu_decode(wl, t, _box_summary(wl, t))
    compare(wl, g, _oracle_box_decode(wl))
