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
