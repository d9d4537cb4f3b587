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
