"""One decode step recorded into a CUDA graph (eta_decode_graph_*): replays
are bit-identical to eta_decode and to one another, every launch reads its
inputs afresh (a new query, new cache contents, new sequence lengths and
thresholds written into the same buffers give the oracle's result for the new
state), and recording can be the first call a process makes."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import workloads
from etatest import compare, gpu_summary, oracle_decode, upload

pytestmark = pytest.mark.gpu

F32, BF16 = workloads.F32, workloads.BF16
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("out", "lse", "admitted_count", "union_count", "union_list", "union_mask")


def _setup(wl, t, summ, impl=eta.ETA_ATTEND_AUTO):
    B, Hq, _ = t["q"].shape
    nb = wl.nb_max
    dev = t["q"].device
    res = {"out": torch.empty_like(t["q"]), "lse": torch.empty((B, Hq), dtype=torch.float32, device=dev),
           "admitted_count": torch.empty((B, Hq), dtype=torch.int32, device=dev),
           "union_count": torch.empty((B, wl.n_kv_heads), dtype=torch.int32, device=dev),
           "union_list": torch.empty((B, wl.n_kv_heads, nb), dtype=torch.int32, device=dev),
           "union_mask": torch.empty((B, wl.n_kv_heads, nb), dtype=torch.int32, device=dev)}
    p = eta.make_params(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, wl.tau_mode, w_tau=t["w_tau"],
                        b_tau=t["b_tau"], c_tau=t["c_tau"], scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a,
                        z=wl.z, n_local_blocks=wl.n_local_blocks, attend_impl=impl, **res)
    ws = eta.alloc_workspace(eta.eta_decode_workspace_size(p))
    p.workspace = ws.data_ptr()
    p.workspace_bytes = ws.numel()
    return p, ws, res


def _host(res, ws):
    torch.cuda.synchronize()
    out = {k: (res[k].float().cpu().numpy() if k == "out" else res[k].cpu().numpy()) for k in KEYS}
    out["status"] = eta.eta_read_device_status(ws)
    return out


def _clear(res):
    for v in res.values():
        v.fill_(0)


CASES = [
    dict(id="tc_bf16_ragged", seed=2, B=3, Hq=16, Hkv=4, d=128, b=64, lens=[3000, 1, 777], dtype=BF16,
         impl=eta.ETA_ATTEND_AUTO),
    dict(id="simt_bf16_ragged", seed=2, B=3, Hq=16, Hkv=4, d=128, b=64, lens=[3000, 1, 777], dtype=BF16,
         impl=eta.ETA_ATTEND_SIMT),
    dict(id="simt_f32_d64", seed=1, B=1, Hq=4, Hkv=4, d=64, b=64, lens=[1000], dtype=F32,
         impl=eta.ETA_ATTEND_AUTO),
]


@pytest.mark.parametrize("c", CASES, ids=[c["id"] for c in CASES])
def test_graph_replay_equals_decode(c):
    wl = workloads.custom(seed=c["seed"], batch=c["B"], n_q_heads=c["Hq"], n_kv_heads=c["Hkv"], head_dim=c["d"],
                          block_size=c["b"], seq_lens=c["lens"], dtype=c["dtype"], tau_bias=2.0, tau_std=1.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    p, ws, res = _setup(wl, t, summ, c["impl"])
    eta.eta_decode(p)
    ref = _host(res, ws)
    assert ref["status"] == eta.ETA_OK
    g = eta.DecodeGraph(p, [ws, *res.values()])
    try:
        for _ in range(3):
            _clear(res)
            g.launch()
            got = _host(res, ws)
            for k in KEYS:
                np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
            assert got["status"] == eta.ETA_OK
    finally:
        g.close()


def test_graph_reads_new_contents_each_launch():
    shape = dict(batch=2, n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=64, dtype=BF16, max_ctx=4096)
    wl1 = workloads.custom(seed=11, seq_lens=[3000, 700], tau_bias=2.0, tau_std=1.0, **shape)
    wl2 = workloads.custom(seed=12, seq_lens=[3001, 4096], tau_bias=1.0, tau_std=0.5, key_kind="cluster", **shape)
    t = upload(wl1)
    summ = gpu_summary(wl1, t)
    p, ws, res = _setup(wl1, t, summ)
    g = eta.DecodeGraph(p, [ws, *res.values(), *[v for v in t.values() if v is not None], *summ.values()])
    try:
        g.launch()
        compare(wl1, _host(res, ws), oracle_decode(wl1))
        # the second state goes into the same buffers; the graph is not rebuilt
        t2 = upload(wl2)
        for name in ("q", "k", "v", "seq", "w_tau", "b_tau"):
            t[name].copy_(t2[name])
        first = torch.zeros(wl2.batch, dtype=torch.int32, device="cuda")
        eta.eta_block_summary_update(t["k"], t["v"], t["seq"], summ, wl2.block_size, first, wl2.nb_max,
                                     wl2.n_q_heads)
        _clear(res)
        g.launch()
        compare(wl2, _host(res, ws), oracle_decode(wl2))
    finally:
        g.close()


def test_graph_as_first_call_of_a_process():
    code = r'''
import sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import learned_threshold_sparse_b200 as eta
import workloads
wl = workloads.custom(seed=5, batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                      seq_lens=[2000], dtype=workloads.BF16, tau_bias=2.0, tau_std=1.0)
q, k, v = wl.q.cuda(), wl.k.cuda(), wl.v.cuda()
seq = torch.tensor(wl.seq_lens, dtype=torch.int32, device="cuda")
w, b = torch.from_numpy(wl.w_tau).cuda(), torch.from_numpy(wl.b_tau).cuda()
summ = eta.alloc_summary(1, 2, wl.max_ctx, 128, 64)
out, lse = torch.empty_like(q), torch.empty((1, 8), dtype=torch.float32, device="cuda")
p = eta.make_params(q, k, v, seq, summ, 64, "learned", w_tau=w, b_tau=b, scale=wl.scale, out=out, lse=lse)
ws = eta.alloc_workspace(eta.eta_decode_workspace_size(p))
p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
torch.cuda.synchronize()
h = eta.eta_decode_graph_create(p)          # the library's first kernel-related call
first = torch.zeros(1, dtype=torch.int32, device="cuda")
eta.eta_block_summary_update(k, v, seq, summ, 64, first, wl.nb_max, 8)
eta.eta_decode_graph_launch(h)
torch.cuda.synchronize()
a = out.clone()
eta.eta_decode(p)
torch.cuda.synchronize()
assert eta.eta_read_device_status(ws) == eta.ETA_OK
assert torch.equal(a, out)
eta.eta_decode_graph_destroy(h)
print("first-call graph ok")
'''
    r = subprocess.run([sys.executable, "-c", code, ROOT], capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "first-call graph ok" in r.stdout


@pytest.mark.parametrize("name", ["c2_single", "c3_long", "c4_max", "c5_batched"])
def test_graph_full_size_equals_decode(name):
    """The launch the bench times (one graph replay per step) at the workloads'
    full sizes gives exactly what eta_decode gives; eta_decode itself is held
    to the oracle at these sizes by the parity suite."""
    wl = workloads.make(name, 0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    p, ws, res = _setup(wl, t, summ)
    eta.eta_decode(p)
    ref = _host(res, ws)
    assert ref["status"] == eta.ETA_OK
    g = eta.DecodeGraph(p, [ws, *res.values()])
    try:
        _clear(res)
        g.launch()
        got = _host(res, ws)
    finally:
        g.close()
    for k in KEYS:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    assert got["status"] == eta.ETA_OK


@pytest.mark.parametrize("mode", ["copies", "direct"])
def test_step_graph_equals_separate_calls(mode):
    """One serving-loop token as one graph leaves the caches, the metadata and
    the host output exactly as separate calls do, token after token.
    copies: input copy from page-locked host memory, append, decode, output
    copy back.  direct: the append reads the new q, k, v rows from
    page-locked host memory itself and the decode stores its output straight
    into page-locked host memory (no copies)."""
    shape = dict(batch=3, n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=64, dtype=BF16, max_ctx=3200)
    wl = workloads.custom(seed=21, seq_lens=[3000, 1, 777], tau_bias=2.0, tau_std=1.0, **shape)
    B, Hq, Hkv, d = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    nq, nkv = B * Hq * d, B * Hkv * d
    host = torch.empty(nq + 2 * nkv, dtype=torch.bfloat16).pin_memory()
    states = []
    for _ in range(2):  # A: separate calls, B: one recorded step
        t = upload(wl)
        summ = gpu_summary(wl, t)
        packed = torch.empty(host.shape, dtype=host.dtype, device="cuda")
        q_in = packed[:nq].view(B, Hq, d)
        k_in, v_in = packed[nq:nq + nkv].view(B, Hkv, d), packed[nq + nkv:].view(B, Hkv, d)
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
        out_h = torch.zeros((B, Hq, d), dtype=torch.bfloat16).pin_memory()
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        states.append(dict(t=t, summ=summ, packed=packed, q_in=q_in, k_in=k_in, v_in=v_in, out=out, lse=lse,
                           out_h=out_h, pos=torch.tensor(wl.seq_lens, dtype=torch.int32, device="cuda")))
    for n, st in enumerate(states):
        direct = n == 1 and mode == "direct"
        st["p"] = eta.make_params(st["q_in"], st["t"]["k"], st["t"]["v"], st["t"]["seq"], st["summ"], wl.block_size,
                                  wl.tau_mode, w_tau=st["t"]["w_tau"], b_tau=st["t"]["b_tau"], scale=wl.scale,
                                  beta=wl.beta, z=wl.z, n_local_blocks=wl.n_local_blocks,
                                  out=st["out_h"] if direct else st["out"], lse=st["lse"])
        st["ws"] = eta.alloc_workspace(eta.eta_decode_workspace_size(st["p"]))
        st["p"].workspace, st["p"].workspace_bytes = st["ws"].data_ptr(), st["ws"].numel()
    a, b = states
    keep = [b["ws"], b["lse"], b["out"], *b["summ"].values()]
    if mode == "direct":
        g = eta.StepGraph(b["p"], k_new=host[nq:nq + nkv].view(B, Hkv, d), v_new=host[nq + nkv:].view(B, Hkv, d),
                          positions=b["pos"], q_new=host[:nq].view(B, Hq, d), tensors=keep + [b["q_in"]])
    else:
        g = eta.StepGraph(b["p"], k_new=b["k_in"], v_new=b["v_in"], positions=b["pos"], h2d=host,
                          h2d_dst=b["packed"], d2h_src=b["out"], d2h=b["out_h"], tensors=keep)
    rng = np.random.default_rng(3)
    try:
        for _ in range(3):
            host.copy_(torch.from_numpy(rng.standard_normal(host.numel()).astype(np.float32)).to(torch.bfloat16))
            for st in (a, b):
                st["t"]["seq"] += 1  # the new token counts before the append
            torch.cuda.synchronize()
            a["packed"].copy_(host, non_blocking=True)
            eta.eta_append_kv(a["t"]["k"], a["t"]["v"], a["t"]["seq"], a["summ"], wl.block_size, a["k_in"],
                              a["v_in"], a["pos"], Hq)
            eta.eta_decode(a["p"])
            a["out_h"].copy_(a["out"], non_blocking=True)
            g.launch()
            torch.cuda.synchronize()
            for st in (a, b):
                assert eta.eta_read_device_status(st["ws"]) == eta.ETA_OK
            assert torch.equal(a["out_h"], b["out_h"])
            assert torch.equal(a["lse"], b["lse"])
            if mode == "direct":
                assert torch.equal(b["q_in"], a["q_in"])  # the queries landed in the decode's q
            assert torch.equal(a["t"]["k"], b["t"]["k"]) and torch.equal(a["t"]["v"], b["t"]["v"])
            for name in a["summ"]:
                assert torch.equal(a["summ"][name], b["summ"][name]), name
            for st in (a, b):
                st["pos"] += 1
    finally:
        g.close()


@pytest.mark.parametrize("nbytes,offset", [(1001, 0), (4096, 3), (16, 0), (70000, 5)])
def test_step_graph_copies_of_any_size_and_alignment(nbytes, offset):
    """The step's input and output copies move exactly their bytes, also for
    sizes that are not a multiple of 16 and for buffers that start off a
    16-byte boundary (the copy kernel's byte path)."""
    wl = workloads.custom(seed=8, batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64, block_size=64, seq_lens=[300],
                          dtype=F32, tau_bias=2.0, tau_std=1.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    p, ws, res = _setup(wl, t, summ)
    rng = np.random.default_rng(nbytes)
    src_h = torch.from_numpy(rng.integers(0, 256, nbytes + offset, dtype=np.uint8)).pin_memory()
    dst_d = torch.zeros(nbytes + offset, dtype=torch.uint8, device="cuda")
    src_d = torch.from_numpy(rng.integers(0, 256, nbytes + offset, dtype=np.uint8)).cuda()
    dst_h = torch.zeros(nbytes + offset, dtype=torch.uint8).pin_memory()
    g = eta.StepGraph(p, h2d=src_h[offset:], h2d_dst=dst_d[offset:], d2h_src=src_d[offset:], d2h=dst_h[offset:],
                      tensors=[ws, *res.values(), src_h, dst_d, src_d, dst_h])
    try:
        g.launch()
        torch.cuda.synchronize()
    finally:
        g.close()
    assert torch.equal(dst_d[offset:].cpu(), src_h[offset:])
    assert torch.equal(dst_h[offset:], src_d[offset:].cpu())
    assert not dst_d[:offset].any() and not dst_h[:offset].any()  # nothing written before the buffers
    assert eta.eta_read_device_status(ws) == eta.ETA_OK


@pytest.mark.parametrize("lwb", [2, 0, -1], ids=["window2", "window0", "no_window"])
def test_step_graph_growing_context_across_block_boundaries(lwb):
    """A serving loop whose context grows one token per step, as the bench's
    end-to-end leg runs it: per token the new lengths and positions are copied
    up from page-locked memory, the append reads the new q, k, v rows from
    page-locked host memory, and the decode stores its output into page-locked
    host memory, all in one recorded graph.  The appends cross block
    boundaries (and start a fresh block); after every token the outputs, the
    admitted sets and the refreshed metadata match the oracle for the state
    reached; with the window of two blocks, of the tail block alone (the block
    a token completes is screened by the very next token), and without a
    window (rescue on)."""
    full = workloads.custom(seed=61, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                            seq_lens=[900, 400], dtype=BF16, tau_bias=2.0, tau_std=1.0,
                            key_kind="cluster").with_params(n_local_blocks=lwb)
    T0 = [700 - 4, 256 - 2]  # the first sequence crosses 704, the second 256
    B, Hq, Hkv, d, b = full.batch, full.n_q_heads, full.n_kv_heads, full.head_dim, full.block_size
    wl = full.with_params(seq_lens=list(T0))
    t = upload(wl)
    for i in range(B):  # the rows to come are written by the appends
        t["k"][i, :, T0[i]:] = 0
        t["v"][i, :, T0[i]:] = 0
    summ = gpu_summary(wl, t)
    nq, nkv = B * Hq * d, B * Hkv * d
    rows_h = torch.empty(nq + 2 * nkv, dtype=torch.bfloat16).pin_memory()
    rows_h[:nq].copy_(full.q.reshape(-1))
    lens_h = torch.zeros(2 * B, dtype=torch.int32).pin_memory()
    lens_d = torch.tensor(T0 + [0] * B, dtype=torch.int32, device="cuda")
    q_in = torch.empty_like(t["q"])
    t2 = dict(t, q=q_in, seq=lens_d[:B])
    p, ws, res = _setup(wl, t2, summ)
    out_h = torch.zeros((B, Hq, d), dtype=torch.bfloat16).pin_memory()
    p.out = out_h.data_ptr()
    g = eta.StepGraph(p, k_new=rows_h[nq:nq + nkv].view(B, Hkv, d), v_new=rows_h[nq + nkv:].view(B, Hkv, d),
                      positions=lens_d[B:], q_new=rows_h[:nq].view(B, Hq, d), h2d=lens_h, h2d_dst=lens_d,
                      tensors=[ws, *res.values(), *summ.values(), q_in, t["k"], t["v"], out_h])
    try:
        for s in range(8):
            lens = [T0[i] + s + 1 for i in range(B)]
            for i in range(B):
                rows_h[nq + i * Hkv * d:nq + (i + 1) * Hkv * d].copy_(full.k[i, :, lens[i] - 1].reshape(-1))
                rows_h[nq + nkv + i * Hkv * d:nq + nkv + (i + 1) * Hkv * d].copy_(full.v[i, :, lens[i] - 1].reshape(-1))
                lens_h[i] = lens[i]
                lens_h[B + i] = lens[i] - 1
            g.launch()
            torch.cuda.synchronize()
            got = _host(res, ws)
            got["out"] = out_h.float().numpy()
            now = full.with_params(seq_lens=lens)
            ref = oracle_decode(now)
            compare(now, got, ref)
            # the refreshed tail metadata is the oracle's
            for i in range(B):
                j = (lens[i] - 1) // b
                np.testing.assert_array_equal(summ["mu"][i, :, j].cpu().numpy(), ref["mu"][i, :, j])
                np.testing.assert_array_equal(summ["sigma"][i, :, j].cpu().numpy(), ref["sigma"][i, :, j])
        for i in range(B):
            n = T0[i] + 8
            assert torch.equal(t["k"][i, :, :n].cpu(), full.k[i, :, :n])
            assert torch.equal(t["v"][i, :, :n].cpu(), full.v[i, :, :n])
    finally:
        g.close()
