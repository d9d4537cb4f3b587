"""FP8 block metadata on the device against the FP8 oracle: codes and scales
bit-exact (the device evaluates the statistics, the scale and each quotient in
float64 and rounds once, as the oracle's definition does; a code may differ
only where the exact quotient lies within a float64 hair of an e4m3 rounding
boundary, counted and printed), M equal or one fp32 step above and a true
bound for the device's own dequantised centroid, the append path refreshing
only the tail block, and whole decode steps screened with FP8 metadata under
the same comparison rules as the fp16 metadata."""
import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import oracle
import workloads
from etatest import assert_bits_equal, compare, gpu_decode, oracle_decode, upload
from oracle import eta_fp8_oracle as fo

pytestmark = pytest.mark.gpu

F32, BF16 = workloads.F32, workloads.BF16


def _fp8_summary(wl, t):
    summ = eta.alloc_summary(wl.batch, wl.n_kv_heads, wl.max_ctx, wl.head_dim, wl.block_size, fmt="fp8")
    first = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    eta.eta_block_summary_update(t["k"], t["v"], t["seq"], summ, wl.block_size, first, wl.nb_max, wl.n_q_heads)
    torch.cuda.synchronize()
    return summ


def _check_blocks(wl, summ, ref, blocks=None):
    got = {k: v.cpu().numpy() for k, v in summ.items()}
    n_exc = 0
    for i, T in enumerate(wl.seq_lens):
        nb = wl.n_blocks(i)
        for g in range(wl.n_kv_heads):
            js = range(nb) if blocks is None else blocks(i)
            for j in js:
                rows = oracle.as_f64(wl.k[i, g, j * wl.block_size:min(T, (j + 1) * wl.block_size)])
                for name, stat in (("mu", rows.mean(axis=0)), ("sigma", rows.std(axis=0))):
                    scl = float(ref[name + "_scale"][i, g, j])
                    assert got[name + "_scale"][i, g, j] == ref[name + "_scale"][i, g, j], (name, i, g, j)
                    n_exc += assert_bits_equal(got[name][i, g, j], ref[name + "_code"][i, g, j], stat / scl,
                                               fo.e4m3_encode, f"{name} codes seq {i} kv {g} block {j}")
                m_g, m_r = got["max_norm"][i, g, j], ref["max_norm"][i, g, j]
                assert m_g == m_r or m_g == np.nextafter(m_r, np.float32(np.inf)), (i, g, j, m_g, m_r)
                mu_dev = fo.e4m3_decode(got["mu"][i, g, j]).astype(np.float64) * float(got["mu_scale"][i, g, j])
                assert np.sqrt(((rows - mu_dev) ** 2).sum(axis=1)).max() <= float(m_g)
    print(f"fp8 codes excused next to a rounding boundary: {n_exc}")


@pytest.mark.parametrize("case", [
    dict(dtype=BF16, d=128, b=64, lens=[1000, 1, 64, 0], kind="cluster"),
    dict(dtype=F32, d=64, b=32, lens=[777]),
    dict(dtype=BF16, d=128, b=128, lens=[3000, 129]),
])
def test_fp8_summary_codes_bit_exact(case):
    wl = workloads.custom(seed=41, batch=len(case["lens"]), n_q_heads=4, n_kv_heads=2, head_dim=case["d"],
                          block_size=case["b"], seq_lens=case["lens"], dtype=case["dtype"],
                          key_kind=case.get("kind", "normal"))
    t = upload(wl)
    _check_blocks(wl, _fp8_summary(wl, t), fo.summarize_fp8(wl.k, wl.seq_lens, wl.block_size))


def test_fp8_append_refreshes_the_tail_block_only():
    wl = workloads.custom(seed=42, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=128, block_size=64,
                          seq_lens=[300, 129], dtype=BF16, max_ctx=400)
    t = upload(wl)
    summ = _fp8_summary(wl, t)
    before = {k: v.clone() for k, v in summ.items()}
    rng = np.random.default_rng(5)
    knew = torch.from_numpy(rng.standard_normal((2, 2, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
    vnew = torch.from_numpy(rng.standard_normal((2, 2, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
    lens = [301, 130]
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    pos = torch.tensor([300, 129], dtype=torch.int32, device="cuda")
    eta.eta_append_kv(t["k"], t["v"], seq, summ, wl.block_size, knew, vnew, pos, wl.n_q_heads)
    torch.cuda.synchronize()
    k_host = t["k"].cpu()
    ref = fo.summarize_fp8(k_host, lens, wl.block_size)
    wl2 = wl.with_params(seq_lens=lens, k=k_host)
    _check_blocks(wl2, summ, ref, blocks=lambda i: [lens[i] // wl.block_size])
    for i in range(2):
        tail = lens[i] // wl.block_size
        for name in ("mu", "sigma", "mu_scale", "sigma_scale", "max_norm"):
            assert torch.equal(summ[name][i, :, :tail], before[name][i, :, :tail]), name


FP8_DECODE = [
    dict(id="g4_bf16_cluster_ragged", seed=2, B=4, Hq=16, Hkv=4, d=128, b=64, lens=[3000, 1, 64, 777],
         dtype=BF16, mode="calibrated", kind="cluster", bias=1.0),
    dict(id="g8_bf16_d64_b32", seed=3, B=1, Hq=16, Hkv=2, d=64, b=32, lens=[2500], dtype=BF16, bias=2.0, std=1.0),
    dict(id="g4_bf16_b128", seed=5, B=1, Hq=8, Hkv=2, d=128, b=128, lens=[9000], dtype=BF16, bias=2.0, std=1.0),
    dict(id="g1_f32_d64_b64", seed=1, B=1, Hq=4, Hkv=4, d=64, b=64, lens=[1000], dtype=F32, bias=2.0, std=1.0),
]


@pytest.mark.parametrize("c", FP8_DECODE, ids=[c["id"] for c in FP8_DECODE])
def test_fp8_decode_parity(c):
    wl = workloads.custom(seed=c["seed"], batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                          head_dim=c["d"], block_size=c["b"], seq_lens=c["lens"], dtype=c["dtype"],
                          tau_mode=c.get("mode", "learned"), key_kind=c.get("kind", "normal"),
                          tau_bias=c["bias"], tau_std=c.get("std", 0.0))
    t = upload(wl)
    g = gpu_decode(wl, t, _fp8_summary(wl, t))
    r = oracle_decode(wl, summary=fo.summarize_fp8(wl.k, wl.seq_lens, wl.block_size))
    compare(wl, g, r)
