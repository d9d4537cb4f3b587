"""The optional step trace (eta_decode_params.trace, include/eta.h): with it
on, every kernel of the step leaves its first-CTA start and last-CTA end, in
the order the step runs them, and the results are bit-identical to a step
without it."""
import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import workloads
from etatest import gpu_summary, upload

pytestmark = pytest.mark.gpu


def _run(wl, t, summ, impl, trace):
    res = eta.decode(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, wl.tau_mode, w_tau=t["w_tau"],
                     b_tau=t["b_tau"], c_tau=t["c_tau"], attend_impl=impl, scale=wl.scale, beta=wl.beta,
                     offset_a=wl.offset_a, z=wl.z, n_local_blocks=wl.n_local_blocks,
                     screen_enabled=wl.screen_enabled, trace=trace)
    torch.cuda.synchronize()
    assert eta.eta_read_device_status(res["workspace"]) == eta.ETA_OK
    return res["out"].cpu(), res["lse"].cpu()


@pytest.mark.parametrize("impl", [eta.ETA_ATTEND_AUTO, eta.ETA_ATTEND_FUSED], ids=["split", "fused"])
def test_trace_order_and_no_effect_on_results(impl):
    wl = workloads.custom(seed=11, batch=2, n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=64,
                          seq_lens=[20000, 7000], dtype="bf16", tau_bias=2.0, tau_std=1.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    tr = torch.zeros(eta.ETA_TRACE_SLOTS, dtype=torch.int64, device="cuda")
    o1, l1 = _run(wl, t, summ, impl, tr)
    o0, l0 = _run(wl, t, summ, impl, None)
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    assert torch.equal(l0, l1)
    tt = eta.trace_times(tr)
    if impl == eta.ETA_ATTEND_FUSED:
        assert tt["fused_first"] <= tt["tile_first"] <= tt["fused_last"]
        assert "screen_first" not in tt and "attend_first" not in tt
    else:
        assert tt["screen_first"] <= tt["screen_last"]
        assert tt["screen_last"] <= tt["attend_first"] + 2000  # the attention kernel passes its wait after the screen
        assert tt["attend_first"] <= tt["tile_first"] <= tt["attend_last"]
        if "merge_first" in tt:
            assert tt["attend_first"] <= tt["merge_first"] <= tt["merge_last"]
        assert "fused_first" not in tt
    span = max(tt.values()) - min(tt.values())
    assert 0 < span < 50_000_000  # nanoseconds: well under 50 ms


def test_trace_rejects_wrong_buffer():
    wl = workloads.custom(seed=12, batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                          seq_lens=[1000], dtype="bf16", tau_bias=2.0, tau_std=1.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    with pytest.raises(ValueError):
        _run(wl, t, summ, eta.ETA_ATTEND_AUTO, torch.zeros(4, dtype=torch.int64, device="cuda"))


def test_serving_step_trace_order():
    """A recorded serving token (input copy kernel, append, decode, output
    copy kernel) with the trace on: every stage leaves its stamps, in the
    order the token runs them."""
    wl = workloads.custom(seed=13, batch=1, n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=64,
                          seq_lens=[5000], dtype="bf16", tau_bias=2.0, tau_std=1.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    B, Hq, Hkv, d = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    T = wl.seq_lens[0]
    tr = torch.zeros(eta.ETA_TRACE_SLOTS, dtype=torch.int64, device="cuda")
    out_d = torch.empty_like(t["q"])
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    p = eta.make_params(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, wl.tau_mode, w_tau=t["w_tau"],
                        b_tau=t["b_tau"], c_tau=t["c_tau"], scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a,
                        z=wl.z, n_local_blocks=wl.n_local_blocks, out=out_d, lse=lse, trace=tr)
    ws = eta.alloc_workspace(eta.eta_decode_workspace_size(p))
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    k_new = t["k"][:, :, T - 1].contiguous()  # the last token again: the cache stays as it is
    v_new = t["v"][:, :, T - 1].contiguous()
    pos_h = torch.tensor([T - 1], dtype=torch.int32).pin_memory()
    pos_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_h = torch.empty((B, Hq, d), dtype=out_d.dtype).pin_memory()
    g = eta.StepGraph(p, k_new=k_new, v_new=v_new, positions=pos_d, h2d=pos_h, h2d_dst=pos_d, d2h_src=out_d,
                      d2h=out_h, tensors=[ws, tr, lse, *summ.values(), t["k"], t["v"], t["q"], t["seq"]])
    try:
        for _ in range(2):
            tr.zero_()
            g.launch()
            torch.cuda.synchronize()
        tt = eta.trace_times(tr)
        order = ["in_first", "in_last", "append_first", "append_last", "screen_first", "screen_last",
                 "attend_first", "tile_first", "attend_last", "out_first", "out_last"]
        missing = [n for n in order if n not in tt]
        assert not missing, missing
        seq = [tt[n] for n in order]
        # each stage starts after the one before it has ended (PDL lets the
        # next kernel's CTAs start early, but only past their wait is stamped)
        assert all(a <= b + 2000 for a, b in zip(seq, seq[1:])), list(zip(order, seq))
        assert torch.equal(out_h, out_d.cpu())
    finally:
        g.close()
