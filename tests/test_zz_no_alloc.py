"""eta_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (it uses the library's fixed device scratch instead of a caller
workspace).  Checked through the C ABI against eta_decode with a workspace on
calls in a row with different shapes (a call after one that ran the rescue
path and left other contents in the shared scratch included), for the status
word it hands back, and for its size limit."""
import ctypes

import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import workloads
from etatest import OUT_TOL, gpu_summary, upload

pytestmark = pytest.mark.gpu


def _case(seed, **kw):
    return workloads.custom(seed=seed, **kw)


def _params(wl, t, summ, out, lse):
    return eta.make_params(t["q"], t["k"], t["v"], t["seq"], summ, wl.block_size, wl.tau_mode, w_tau=t["w_tau"],
                           b_tau=t["b_tau"], c_tau=t["c_tau"], scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a,
                           z=wl.z, n_local_blocks=wl.n_local_blocks, out=out, lse=lse)


def test_noalloc_matches_workspace_entry_point_twice():
    first = _case(31, batch=3, n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=64, seq_lens=[3000, 130, 1777],
                  dtype=workloads.BF16, tau_mode="calibrated", key_kind="cluster", tau_bias=1.0)
    rescue = _case(32, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=64, block_size=32, seq_lens=[900, 47],
                   dtype=workloads.F32, tau_bias=1e6).with_params(n_local_blocks=-1)
    # the third call reuses the first shape after the rescue call, so stale
    # rescue counters and chunk lists from a different shape sit in the scratch
    lib = eta.library()
    stream = torch.cuda.current_stream()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for wl in (first, rescue, first):
        t = upload(wl)
        summ = gpu_summary(wl, t)
        ref_out = torch.empty_like(t["q"])
        ref_lse = torch.empty(wl.batch, wl.n_q_heads, dtype=torch.float32, device="cuda")
        p_ref = _params(wl, t, summ, ref_out, ref_lse)
        ws = eta.alloc_workspace(eta.eta_decode_workspace_size(p_ref))
        p_ref.workspace = ws.data_ptr()
        p_ref.workspace_bytes = ws.numel()
        eta.eta_decode(p_ref)
        out = torch.full_like(t["q"], float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        p = _params(wl, t, summ, out, lse)  # no workspace: the entry point ignores it anyway
        status.fill_(-1)
        rc = lib.eta_decode_noalloc(ctypes.byref(p), ctypes.c_void_p(status.data_ptr()),
                                    ctypes.c_void_p(stream.cuda_stream))
        assert rc == eta.ETA_OK, eta.eta_status_string(rc)
        torch.cuda.synchronize()
        assert status.item() == 0
        err = (out.float() - ref_out.float()).abs().max().item()
        assert err <= OUT_TOL[wl.dtype], err
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=1e-5, atol=1e-5)


def test_noalloc_hands_back_the_device_status():
    # a sequence length past the cache capacity is clamped on the device and
    # reported in the status word; the next clean call reports 0
    wl = _case(33, batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64, block_size=64, seq_lens=[256],
               dtype=workloads.BF16, tau_bias=2.0)
    t = upload(wl)
    summ = gpu_summary(wl, t)
    out = torch.empty_like(t["q"])
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t["seq"].fill_(257)
    eta.eta_decode_noalloc(_params(wl, t, summ, out, None), device_status=status)
    torch.cuda.synchronize()
    assert status.item() == eta.DEVICE_STATUS_RANGE
    t["seq"].fill_(256)
    eta.eta_decode_noalloc(_params(wl, t, summ, out, None), device_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    fake = 1 << 20  # never dereferenced: the size check fails before any launch
    p = eta.eta_decode_params()
    p.cache = eta.eta_cache_desc(256, 64, 8, 128, 64, 131072, eta.ETA_BF16, fake, fake, fake)
    p.summary = eta.eta_summary_desc(fake, fake, fake)
    p.q = fake
    p.out = fake
    p.tau_mode = eta.ETA_TAU_CALIBRATED
    p.c_tau = fake
    p.scale, p.beta, p.z, p.n_local_blocks, p.screen_enabled = 0.088, 5.0, 2.0, 2, 1
    need = eta.eta_decode_workspace_size(p)
    assert need > eta.NOALLOC_SCRATCH_BYTES
    rc = eta.library().eta_decode_noalloc(ctypes.byref(p), None, None)
    assert rc == eta.ETA_ERR_WORKSPACE
