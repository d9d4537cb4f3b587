"""Failure reporting without a GPU fault: a bounded device-side wait that
nothing completes gives up after its cycle limit, the status word in the
workspace reports ETA_ERR_DEVICE_TIMEOUT (and is cleared by the read), and the
context stays usable for the next decode step."""
import pytest

import learned_threshold_sparse_b200 as eta
import workloads
from etatest import compare, gpu_decode, oracle_decode

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = eta.alloc_workspace(256)
    eta.eta_diag_wait_timeout(ws)
    assert eta.eta_read_device_status(ws) == eta.ETA_ERR_DEVICE_TIMEOUT
    assert eta.eta_read_device_status(ws) == eta.ETA_OK  # the read cleared the word
    wl = workloads.custom(seed=1, batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64, block_size=64, seq_lens=[1000],
                          dtype=workloads.F32, tau_bias=2.0, tau_std=1.0)
    compare(wl, gpu_decode(wl), oracle_decode(wl))
