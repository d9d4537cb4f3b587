"""Offline calibration on the device against the oracle: the weighted causal
logit histogram (total weight = query rows; bin contents equal up to logits
that sit within fp32 rounding of a bin edge), accumulation across calls, and
the constants solved from the device histogram within one bin width of the
oracle's exact constants, reaching the target density on the same data."""
import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import workloads
from oracle import eta_calib_oracle as co

pytestmark = pytest.mark.gpu

LO, HI, NB = -6.0, 6.0, 1200


def _case(seed, B, Hq, Hkv, T, d, dtype=torch.bfloat16):
    c = workloads.prefill_case(seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv, seq_len=T, head_dim=d)
    if dtype == torch.float32:
        return c.q.float(), c.k.float(), c.scale
    return c.q, c.k, c.scale


@pytest.mark.parametrize("shape", [(2, 4, 2, 300, 128, torch.bfloat16), (1, 2, 2, 190, 64, torch.float32),
                                   (1, 8, 2, 1024, 128, torch.bfloat16)])
def test_histogram_and_constants(shape):
    B, Hq, Hkv, T, d, dt = shape
    q, k, scale = _case(31, B, Hq, Hkv, T, d, dt)
    hist = eta.calibration_histogram(q.cuda(), k.cuda(), T, scale=scale, lo=LO, hi=HI, nbins=NB)
    torch.cuda.synchronize()
    got = hist.cpu().numpy()
    logits = co.calibration_logits(q, k, T, scale)
    targets = [0.1, 0.38, 0.7]
    for h in range(Hq):
        S, w = logits[h]
        ref = co.histogram(S, w, LO, HI, NB)
        assert abs(got[h].sum() - B * T) <= 1e-5 * B * T
        assert np.abs(got[h] - ref).sum() <= 2e-3 * B * T
        for p in targets:
            c_dev = eta.calibrate_constants(hist[h:h + 1], LO, HI, p)[0]
            c_ex = co.exact_constant(S, w, p)
            assert abs(c_dev - c_ex) <= (HI - LO) / NB + 1e-3, (h, p, c_dev, c_ex)
            # the calibrated constant reaches the target on the calibration data
            assert abs(co.density(S, w, c_dev) - p) <= 0.01


def test_histogram_accumulates_across_calls():
    q, k, scale = _case(32, 1, 2, 1, 200, 128)
    q, k = q.cuda(), k.cuda()
    h1 = eta.calibration_histogram(q, k, 200, scale=scale, lo=LO, hi=HI, nbins=NB)
    once = h1.clone()
    eta.calibration_histogram(q, k, 200, scale=scale, lo=LO, hi=HI, nbins=NB, hist=h1)
    torch.cuda.synchronize()
    np.testing.assert_allclose(h1.cpu().numpy(), 2 * once.cpu().numpy(), rtol=1e-6, atol=1e-9)
