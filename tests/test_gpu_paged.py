"""Paged KV cache: the same cache scattered into a pool of pages (one KV block
per page, a shuffled page table, unused pages and rows past each sequence's
end filled with NaN) must give bit-identical metadata, decode outputs and
selections to the contiguous layout, for both attention kernels and both
metadata formats; the contiguous results are themselves checked against the
oracle by the parity suite, and once more here."""
import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import workloads
from etatest import compare, oracle_decode, upload

pytestmark = pytest.mark.gpu

F32, BF16 = workloads.F32, workloads.BF16

CASES = [
    dict(id="tc_g4_bf16_b64_ragged", seed=2, B=4, Hq=16, Hkv=4, d=128, b=64, lens=[3000, 1, 64, 777],
         dtype=BF16, mode="calibrated", kind="cluster", bias=1.0),
    dict(id="tc_g4_bf16_b128", seed=5, B=1, Hq=8, Hkv=2, d=128, b=128, lens=[9000], dtype=BF16, bias=2.0, std=1.0),
    dict(id="simt_g1_f32_d64", seed=1, B=1, Hq=4, Hkv=4, d=64, b=64, lens=[1000], dtype=F32, bias=2.0, std=1.0),
    dict(id="simt_g8_bf16_d64_b32", seed=3, B=1, Hq=16, Hkv=2, d=64, b=32, lens=[2500], dtype=BF16, bias=2.0,
         std=1.0),
    dict(id="ctx_not_block_multiple", seed=6, B=2, Hq=8, Hkv=2, d=128, b=64, lens=[1000, 999], dtype=BF16,
         bias=2.0, std=1.0, max_ctx=1000),
]


def _wl(c):
    return workloads.custom(seed=c["seed"], batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                            head_dim=c["d"], block_size=c["b"], seq_lens=c["lens"], dtype=c["dtype"],
                            tau_mode=c.get("mode", "learned"), key_kind=c.get("kind", "normal"),
                            tau_bias=c["bias"], tau_std=c.get("std", 0.0), max_ctx=c.get("max_ctx"))


def _paged(wl, t, seed=0, extra=5):
    """Scatter the contiguous cache into shuffled pages; returns (k_pool,
    v_pool, table)."""
    b, d = wl.block_size, wl.head_dim
    nbs = [wl.n_blocks(i) for i in range(wl.batch)]
    P = sum(nbs) + extra
    perm = np.random.default_rng(seed).permutation(P)
    kd = t["k"].dtype
    kp = torch.full((P, wl.n_kv_heads, b, d), float("nan"), dtype=kd, device="cuda")
    vp = torch.full_like(kp, float("nan"))
    table = torch.full((wl.batch, wl.nb_max), -1, dtype=torch.int32)
    x = 0
    for i, T in enumerate(wl.seq_lens):
        for j in range(nbs[i]):
            page = int(perm[x])
            x += 1
            table[i, j] = page
            lo, hi = j * b, min(T, (j + 1) * b)  # rows past the sequence end stay NaN
            kp[page, :, :hi - lo] = t["k"][i, :, lo:hi]
            vp[page, :, :hi - lo] = t["v"][i, :, lo:hi]
    return kp, vp, table.cuda()


def _summ(wl, k, v, seq, fmt, table=None):
    s = eta.alloc_summary(wl.batch, wl.n_kv_heads, wl.max_ctx, wl.head_dim, wl.block_size, fmt=fmt)
    first = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    eta.eta_block_summary_update(k, v, seq, s, wl.block_size, first, wl.nb_max, wl.n_q_heads, block_table=table)
    return s


def _decode(wl, t, k, v, summ, table=None, impl=eta.ETA_ATTEND_AUTO):
    r = eta.decode(t["q"], k, v, t["seq"], summ, wl.block_size, wl.tau_mode, w_tau=t["w_tau"], b_tau=t["b_tau"],
                   c_tau=t["c_tau"], scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
                   n_local_blocks=wl.n_local_blocks, attend_impl=impl, selection=True, block_table=table)
    torch.cuda.synchronize()
    assert eta.eta_read_device_status(r["workspace"]) == eta.ETA_OK
    return {k2: v2.cpu() for k2, v2 in r.items() if k2 != "workspace"}


@pytest.mark.parametrize("fmt", ["fp16", "fp8"])
@pytest.mark.parametrize("c", CASES, ids=[c["id"] for c in CASES])
def test_paged_equals_contiguous(c, fmt):
    wl = _wl(c)
    t = upload(wl)
    kp, vp, table = _paged(wl, t, seed=c["seed"])
    s_c = _summ(wl, t["k"], t["v"], t["seq"], fmt)
    s_p = _summ(wl, kp, vp, t["seq"], fmt, table)
    for name in s_c:
        for i in range(wl.batch):
            nb = wl.n_blocks(i)
            assert torch.equal(s_c[name][i, :, :nb].cpu(), s_p[name][i, :, :nb].cpu()), name
    impls = [eta.ETA_ATTEND_AUTO] + ([eta.ETA_ATTEND_SIMT] if c["id"].startswith("tc") else [])
    for impl in impls:
        a = _decode(wl, t, t["k"], t["v"], s_c, impl=impl)
        p = _decode(wl, t, kp, vp, s_p, table, impl=impl)
        for name in a:
            assert torch.equal(a[name], p[name]), (impl, name)


def test_paged_against_the_oracle():
    wl = _wl(CASES[0])
    t = upload(wl)
    kp, vp, table = _paged(wl, t, seed=9)
    s_p = _summ(wl, kp, vp, t["seq"], "fp16", table)
    g = _decode(wl, t, kp, vp, s_p, table)
    g = {k: (v.float().numpy() if k == "out" else v.numpy()) for k, v in g.items()}
    g["status"] = eta.ETA_OK
    compare(wl, g, oracle_decode(wl))


def test_paged_append_matches_contiguous():
    wl = workloads.custom(seed=44, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                          seq_lens=[300, 129], dtype=BF16, max_ctx=448)
    t = upload(wl)
    kp, vp, table = _paged(wl, t, seed=4, extra=4)
    # pages for the blocks the appends reach (block 4 of sequence 0 exists; 129 -> block 2 exists)
    s_c = _summ(wl, t["k"], t["v"], t["seq"], "fp16")
    s_p = _summ(wl, kp, vp, t["seq"], "fp16", table)
    rng = np.random.default_rng(8)
    knew = torch.from_numpy(rng.standard_normal((2, 2, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
    vnew = torch.from_numpy(rng.standard_normal((2, 2, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
    seq = torch.tensor([301, 130], dtype=torch.int32, device="cuda")
    pos = torch.tensor([300, 129], dtype=torch.int32, device="cuda")
    eta.eta_append_kv(t["k"], t["v"], seq, s_c, 64, knew, vnew, pos, 8)
    eta.eta_append_kv(kp, vp, seq, s_p, 64, knew, vnew, pos, 8, block_table=table)
    torch.cuda.synchronize()
    tab = table.cpu()
    for i, p_ in enumerate([300, 129]):
        page = int(tab[i, p_ // 64])
        assert torch.equal(kp[page, :, p_ % 64], t["k"][i, :, p_])
        assert torch.equal(vp[page, :, p_ % 64], t["v"][i, :, p_])
    for name in s_c:
        for i, n in enumerate([301, 130]):
            nb = (n + 63) // 64
            assert torch.equal(s_c[name][i, :, :nb], s_p[name][i, :, :nb]), name


def test_out_of_range_page_is_reported():
    wl = _wl(CASES[0])
    t = upload(wl)
    kp, vp, table = _paged(wl, t, seed=3)
    s_p = _summ(wl, kp, vp, t["seq"], "fp16", table)
    bad = table.clone()
    nb0 = wl.n_blocks(0)
    bad[0, nb0 - 1] = kp.shape[0] + 3  # the always-loaded tail block of sequence 0
    r = eta.decode(t["q"], kp, vp, t["seq"], s_p, wl.block_size, wl.tau_mode, c_tau=t["c_tau"], scale=wl.scale,
                   beta=wl.beta, z=wl.z, n_local_blocks=wl.n_local_blocks, block_table=bad)
    torch.cuda.synchronize()
    assert eta.eta_read_device_status(r["workspace"]) == eta.ETA_ERR_DEVICE_RANGE
