"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on
the same seeded inputs.  Small cases span several KV blocks, several screen
chunks and ragged tails; the workload configurations run at full size."""
import math

import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import oracle
import workloads
from etatest import (assert_summary_bit_exact, compare, gpu_admitted, gpu_decode, gpu_summary, min_margin_over_bound,
                     oracle_decode, oracle_screen_on, upload)

pytestmark = pytest.mark.gpu

F32, BF16 = workloads.F32, workloads.BF16


# ------------------------------------------------------------ summaries

@pytest.mark.parametrize("case", [
    dict(dtype=F32, d=64, b=64, lens=[4096]),
    dict(dtype=BF16, d=128, b=64, lens=[1000, 1, 64, 0]),
    dict(dtype=BF16, d=64, b=128, lens=[777]),
    dict(dtype=F32, d=128, b=16, lens=[333, 16]),
    dict(dtype=BF16, d=128, b=32, lens=[2048], kind="cluster"),
])
def test_block_summary_parity(case):
    # bit-exact: the device evaluates mean, spread and distances in float64
    # and rounds once, as the oracle does
    wl = workloads.custom(seed=21, batch=len(case["lens"]), n_q_heads=4, n_kv_heads=2, head_dim=case["d"],
                          block_size=case["b"], seq_lens=case["lens"], dtype=case["dtype"],
                          key_kind=case.get("kind", "normal"))
    t = upload(wl)
    summ = {k: v.cpu().numpy() for k, v in gpu_summary(wl, t).items()}
    ref = oracle.summarize(wl.k, wl.seq_lens, wl.block_size)
    assert_summary_bit_exact(wl, summ, ref)


def test_summary_append_touches_only_tail_block():
    wl = workloads.custom(seed=3, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=128, block_size=64,
                          seq_lens=[700, 640], dtype=BF16, max_ctx=800)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    before = {k: v.clone() for k, v in summ.items()}
    # append one token to each sequence (new K rows), then refresh one block
    t["k"][0, :, 700] = 1.5
    t["k"][1, :, 640] = -0.75
    t["seq"] = torch.tensor([701, 641], dtype=torch.int32, device="cuda")
    first = torch.tensor([700, 640], dtype=torch.int32, device="cuda")
    eta.eta_block_summary_update(t["k"], t["v"], t["seq"], summ, 64, first, 1, 4)
    torch.cuda.synchronize()
    k_new = wl.k.clone()
    k_new[0, :, 700] = 1.5
    k_new[1, :, 640] = -0.75
    ref = oracle.summarize(k_new, [701, 641], 64)
    assert_summary_bit_exact(wl.with_params(k=k_new, seq_lens=[701, 641]), {k: v.cpu().numpy() for k, v in summ.items()},
                             ref, blocks=lambda i: [10])
    # untouched blocks keep their bytes
    assert torch.equal(summ["mu"][0, :, :10], before["mu"][0, :, :10])
    assert torch.equal(summ["max_norm"][1, :, :10], before["max_norm"][1, :, :10])


@pytest.mark.parametrize("dtype,d,b", [(BF16, 128, 64), (F32, 64, 128), (BF16, 64, 32)])
def test_append_kv_writes_rows_and_refreshes_block(dtype, d, b):
    wl = workloads.custom(seed=13, batch=3, n_q_heads=4, n_kv_heads=2, head_dim=d, block_size=b,
                          seq_lens=[700, 640, 300], dtype=dtype, max_ctx=800)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    before = {k: v.clone() for k, v in summ.items()}
    gen = torch.Generator().manual_seed(7)
    knew = torch.randn(3, 2, d, generator=gen).to(wl.torch_dtype)
    vnew = torch.randn(3, 2, d, generator=gen).to(wl.torch_dtype)
    pos = [700, 640, 800]  # the third position is outside the cache: nothing written
    new_lens = [701, 641, 300]
    t["seq"] = torch.tensor(new_lens, dtype=torch.int32, device="cuda")
    eta.eta_append_kv(t["k"], t["v"], t["seq"], summ, b, knew.cuda(), vnew.cuda(),
                      torch.tensor(pos, dtype=torch.int32, device="cuda"), 4)
    torch.cuda.synchronize()
    k_ref, v_ref = wl.k.clone(), wl.v.clone()
    for i in range(2):
        k_ref[i, :, pos[i]] = knew[i]
        v_ref[i, :, pos[i]] = vnew[i]
    assert torch.equal(t["k"].cpu(), k_ref) and torch.equal(t["v"].cpu(), v_ref)
    ref = oracle.summarize(k_ref, new_lens, b)
    assert_summary_bit_exact(wl.with_params(k=k_ref, seq_lens=new_lens), {k: v.cpu().numpy() for k, v in summ.items()},
                             ref, blocks=lambda i: [pos[i] // b] if i < 2 else [])
    for i in range(2):
        j = pos[i] // b
        assert torch.equal(summ["mu"][i, :, :j], before["mu"][i, :, :j])
    assert torch.equal(summ["mu"][2], before["mu"][2]) and torch.equal(summ["max_norm"][2], before["max_norm"][2])


# ------------------------------------------------------------ decode, small

SMALL = [
    dict(id="g1_f32_d64_b64", seed=1, B=1, Hq=4, Hkv=4, d=64, b=64, lens=[1000], dtype=F32, bias=2.0, std=1.0),
    dict(id="g4_bf16_cluster_ragged", seed=2, B=4, Hq=16, Hkv=4, d=128, b=64, lens=[3000, 1, 64, 777],
         dtype=BF16, mode="calibrated", kind="cluster", bias=1.0),
    dict(id="g8_bf16_d64_b32", seed=3, B=1, Hq=16, Hkv=2, d=64, b=32, lens=[2500], dtype=BF16, bias=2.0, std=1.0),
    dict(id="g2_f32_d128_b16_empty_seq", seed=4, B=2, Hq=4, Hkv=2, d=128, b=16, lens=[400, 0], dtype=F32,
         bias=2.0, std=1.0),
    dict(id="g4_bf16_b128", seed=5, B=1, Hq=8, Hkv=2, d=128, b=128, lens=[9000], dtype=BF16, bias=2.0, std=1.0),
    dict(id="g4_bf16_ctx_not_block_multiple", seed=6, B=2, Hq=8, Hkv=2, d=128, b=64, lens=[1000, 999],
         dtype=BF16, bias=2.0, std=1.0, max_ctx=1000),
    dict(id="g2_bf16_d64_b16_long", seed=7, B=1, Hq=4, Hkv=2, d=64, b=16, lens=[6000], dtype=BF16,
         mode="calibrated", kind="cluster", bias=0.8),
]


def _small(c):
    return workloads.custom(seed=c["seed"], batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"],
                            head_dim=c["d"], block_size=c["b"], seq_lens=c["lens"], dtype=c["dtype"],
                            tau_mode=c.get("mode", "learned"), key_kind=c.get("kind", "normal"),
                            tau_bias=c["bias"], tau_std=c.get("std", 0.0), max_ctx=c.get("max_ctx"))


@pytest.mark.parametrize("c", SMALL, ids=[c["id"] for c in SMALL])
def test_decode_parity_small(c):
    wl = _small(c)
    g = gpu_decode(wl)
    r = oracle_decode(wl)
    compare(wl, g, r)
    dens = g["union_count"].sum() / max(1, sum(wl.n_blocks(i) for i in range(wl.batch)) * wl.n_kv_heads)
    assert 0.0 < dens <= 1.0


TC_CASES = [c for c in SMALL if c["dtype"] == BF16 and c["d"] == 128 and c["b"] in (64, 128)
            and c["Hq"] // c["Hkv"] in (2, 4, 8)]


@pytest.mark.parametrize("impl", [eta.ETA_ATTEND_SIMT, eta.ETA_ATTEND_TC, eta.ETA_ATTEND_FUSED],
                         ids=["simt", "tc", "fused"])
@pytest.mark.parametrize("c", TC_CASES, ids=[c["id"] for c in TC_CASES])
def test_decode_parity_each_attention_kernel(c, impl):
    wl = _small(c)
    g = gpu_decode(wl, attend_impl=impl)
    r = oracle_decode(wl)
    compare(wl, g, r)


def test_tc_kernel_rejects_unsupported_shape():
    wl = _small(SMALL[0])  # fp32, d 64, no GQA
    t = upload(wl)
    summ = gpu_summary(wl, t)
    with pytest.raises(eta.EtaError) as e:
        eta.decode(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, "learned", w_tau=t["w_tau"],
                   b_tau=t["b_tau"], attend_impl=eta.ETA_ATTEND_TC)
    assert e.value.code == eta.ETA_ERR_UNSUPPORTED


VARIANTS = [
    dict(id="screen_off", screen_enabled=False),
    dict(id="strict_z_inf", z=math.inf),
    dict(id="offset_a_0.4", offset_a=0.4),
    dict(id="lwb0", n_local_blocks=0),
    dict(id="lwb_large", n_local_blocks=100),
    dict(id="no_window", n_local_blocks=-1),
    dict(id="beta1_z3", beta=1.0, z=3.0),
]


@pytest.mark.parametrize("v", VARIANTS, ids=[v["id"] for v in VARIANTS])
def test_decode_parity_variants(v):
    over = {k: val for k, val in v.items() if k != "id"}
    wl = _small(SMALL[1]).with_params(**over)
    g = gpu_decode(wl)
    r = oracle_decode(wl)
    compare(wl, g, r)
    if v["id"] == "screen_off":
        assert np.all(g["union_count"] == [[wl.n_blocks(i)] * wl.n_kv_heads for i in range(wl.batch)])


def test_rescue_admits_argmax_when_everything_is_pruned():
    wl = workloads.custom(seed=8, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                          seq_lens=[5000, 300], dtype=BF16, tau_bias=1e6).with_params(n_local_blocks=-1)
    g = gpu_decode(wl)
    r = oracle_decode(wl)
    assert r["rescued"].all()
    compare(wl, g, r)
    assert np.all(g["admitted_count"] == 1)


def test_start_dense_init_is_dense_attention():
    # W_tau = 0, b_tau = -8 (section 2.1): every block admitted, and the output
    # equals the screen-off path.
    wl = workloads.custom(seed=9, batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                          seq_lens=[4000], dtype=BF16, tau_bias=-8.0)
    g = gpu_decode(wl)
    g_off = gpu_decode(wl, screen_enabled=False)
    assert np.all(g["union_count"] == 63)
    np.testing.assert_array_equal(g["out"], g_off["out"])


def test_seq_len_out_of_range_reported():
    wl = workloads.custom(seed=10, batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64, block_size=64,
                          seq_lens=[256], dtype=BF16, tau_bias=2.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    t["seq"] = torch.tensor([257], dtype=torch.int32, device="cuda")
    res = eta.decode(t["q"], t["k"], t["v"], t["seq"], summ, 64, "learned", w_tau=t["w_tau"], b_tau=t["b_tau"])
    assert eta.eta_read_device_status(res["workspace"]) == eta.ETA_ERR_DEVICE_RANGE
    assert eta.eta_read_device_status(res["workspace"]) == eta.ETA_OK  # cleared by the read


def test_workspace_too_small_rejected():
    wl = _small(SMALL[0])
    t = upload(wl)
    summ = gpu_summary(wl, t)
    out = torch.empty_like(t["q"])
    p = eta.make_params(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, "learned", w_tau=t["w_tau"],
                        b_tau=t["b_tau"], out=out)
    need = eta.eta_decode_workspace_size(p)
    ws = eta.alloc_workspace(need)
    p.workspace = ws.data_ptr()
    p.workspace_bytes = need - 256
    with pytest.raises(eta.EtaError) as e:
        eta.eta_decode(p)
    assert e.value.code == eta.ETA_ERR_WORKSPACE


@pytest.mark.parametrize("c", TC_CASES, ids=[c["id"] for c in TC_CASES])
def test_fused_and_split_kernels_agree(c):
    # the same admitted sets, outputs within rounding of each other (the
    # partials are split differently: per chunk vs per attention CTA)
    wl = _small(c)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    f = gpu_decode(wl, t, summ, attend_impl=eta.ETA_ATTEND_FUSED)
    sp = gpu_decode(wl, t, summ, attend_impl=eta.ETA_ATTEND_TC)
    for k in ("union_list", "union_mask", "union_count", "admitted_count"):
        np.testing.assert_array_equal(f[k], sp[k], err_msg=k)
    # both are within the oracle tolerances; P is rounded to bf16 over a
    # different tile packing, so they may differ by up to those
    assert np.abs(f["out"] - sp["out"]).max() <= 2e-2
    np.testing.assert_allclose(f["lse"], sp["lse"], rtol=2e-3, atol=2e-3)


def test_simt_and_auto_agree():
    wl = _small(SMALL[1])
    t = upload(wl)
    summ = gpu_summary(wl, t)
    a = gpu_decode(wl, t, summ, attend_impl=eta.ETA_ATTEND_AUTO)
    b = gpu_decode(wl, t, summ, attend_impl=eta.ETA_ATTEND_SIMT)
    np.testing.assert_array_equal(a["union_list"], b["union_list"])
    assert np.abs(a["out"] - b["out"]).max() <= 2e-2


def test_workspace_reuse_across_shapes():
    # A workspace keeps the previous call's bytes; nothing stale may leak into
    # the next call (tiny problems leave most attention CTAs without units).
    a = workloads.custom(seed=41, batch=3, n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=64,
                         seq_lens=[3000, 130, 1777], dtype=BF16, tau_mode="calibrated", key_kind="cluster",
                         tau_bias=1.0)
    b = workloads.custom(seed=42, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=64, block_size=32,
                         seq_lens=[900, 47], dtype=F32, tau_bias=1e6).with_params(n_local_blocks=-1)
    ws = eta.alloc_workspace(64 << 20)
    ws.fill_(0x7f)  # non-zero garbage everywhere after the control region (zero before first use)
    ws[:eta.WORKSPACE_CONTROL_BYTES].zero_()
    for wl, impl in ((a, eta.ETA_ATTEND_AUTO), (b, eta.ETA_ATTEND_AUTO), (a, eta.ETA_ATTEND_FUSED),
                     (b, eta.ETA_ATTEND_AUTO), (a, eta.ETA_ATTEND_FUSED), (a, eta.ETA_ATTEND_AUTO)):
        t = upload(wl)
        summ = gpu_summary(wl, t)
        res = eta.decode(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, wl.tau_mode, w_tau=t["w_tau"],
                         b_tau=t["b_tau"], c_tau=t["c_tau"], n_local_blocks=wl.n_local_blocks, selection=True,
                         workspace=ws, attend_impl=impl)
        torch.cuda.synchronize()
        g = {k: v.float().cpu().numpy() if k == "out" else v.cpu().numpy()
             for k, v in res.items() if k != "workspace"}
        g["status"] = eta.eta_read_device_status(ws)
        compare(wl, g, oracle_decode(wl))


def test_repeat_calls_are_deterministic():
    wl = _small(SMALL[4])
    t = upload(wl)
    summ = gpu_summary(wl, t)
    a = gpu_decode(wl, t, summ)
    b = gpu_decode(wl, t, summ)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


# ------------------------------------------------------------ full configs

@pytest.mark.parametrize("name", ["c1_tiny", "c2_single", "c3_long", "c4_max", "c5_batched"])
def test_config_parity_full_size(name):
    # The workloads are guard-banded (every screened block's |Score - tau~|
    # >= 1e-4, far above the fp32 evaluation error), so the admitted sets must
    # be identical with no allowance, both against the oracle's own screen
    # and against the oracle's screen evaluated on the device's metadata.
    wl = workloads.make(name, 0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    g = gpu_decode(wl, t, summ)
    r = oracle_decode(wl)
    assert_summary_bit_exact(wl, g["summary"], r)
    ratio = min_margin_over_bound(wl, r)
    print(f"{name}: smallest margin / fp32 error bound = {ratio:.1f}")
    if name != "c1_tiny":
        assert ratio > 1.0
    strict = ratio > 1.0
    n_amb = compare(wl, g, r, strict=strict)
    assert n_amb == 0
    np.testing.assert_array_equal(gpu_admitted(wl, g), oracle_screen_on(wl, g["summary"], r))
    if wl.dtype == BF16 and wl.head_dim == 128:
        # the fused screen + attention + merge kernel on the same state
        gf = gpu_decode(wl, t, summ, attend_impl=eta.ETA_ATTEND_FUSED)
        assert compare(wl, gf, r, strict=strict) == 0
    if wl.planted:
        adm = r["admitted"]
        for (i, h), blocks in wl.planted.items():
            assert adm[i, h, blocks].all()
    if wl.target_union_density is not None:
        dd = oracle.densities(r, wl.seq_lens, wl.block_size)
        assert abs(dd["union"].mean() - wl.target_union_density) < 0.03
