"""Parity of the tensor-core causal forward pass (eta_prefill, through the C
ABI) with the fp64 CPU oracle of the same pass, element by element.

Tolerances: outputs are bf16 (one rounding of a convex combination of bf16
values: 2^-8 relative) after fp32 accumulation of bf16-rounded weights and a
gate computed with the hardware tanh (about 2^-11 relative); the output bound
is 2e-2 absolute + 2e-2 relative, the log-sum-exp 2e-2 absolute, the gate sum
5e-3 relative + 2e-2 absolute.
"""
import numpy as np
import pytest
import torch

import learned_threshold_sparse_b200 as eta
import workloads
from oracle import eta_prefill_oracle as po

pytestmark = pytest.mark.gpu

OUT_ATOL, OUT_RTOL = 2e-2, 2e-2
LSE_ATOL = 2e-2
GATE_RTOL, GATE_ATOL = 5e-3, 2e-2


def _run(case):
    dev = "cuda"
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    opt = lambda x: None if x is None else torch.from_numpy(x).to(dev)
    r = eta.prefill(q, k, v, case.seq_len, case.tau_mode, w_tau=opt(case.w_tau), b_tau=opt(case.b_tau),
                    c_tau=opt(case.c_tau), scale=case.scale, beta=case.beta, offset_a=case.offset_a)
    torch.cuda.synchronize()
    assert eta.eta_read_device_status(r["workspace"]) == eta.ETA_OK
    return {n: r[n].float().cpu().numpy() for n in ("out", "lse", "gate_sum")}


def _oracle(case):
    T = case.seq_len
    return po.prefill(case.q, case.k[:, :, :T], case.v[:, :, :T], T, case.tau_mode, w_tau=case.w_tau,
                      b_tau=case.b_tau, c_tau=case.c_tau, scale=case.scale, beta=case.beta,
                      offset_a=case.offset_a)


def _compare(got, ref):
    np.testing.assert_allclose(got["out"], ref["out"], rtol=OUT_RTOL, atol=OUT_ATOL)
    np.testing.assert_allclose(got["lse"], ref["lse"], rtol=0, atol=LSE_ATOL)
    np.testing.assert_allclose(got["gate_sum"], ref["gate_sum"], rtol=GATE_RTOL, atol=GATE_ATOL)


@pytest.mark.parametrize("T", [1, 5, 127, 128, 129, 300])
def test_prefill_lengths(T):
    case = workloads.prefill_case(T, batch=1, n_q_heads=4, n_kv_heads=1, seq_len=T)
    _compare(_run(case), _oracle(case))


def test_prefill_batch_gqa_calibrated():
    case = workloads.prefill_case(11, batch=2, n_q_heads=8, n_kv_heads=2, seq_len=261, tau_mode="calibrated",
                                  tau_bias=0.3, offset_a=0.4)
    _compare(_run(case), _oracle(case))


def test_prefill_group_of_one():
    case = workloads.prefill_case(12, batch=2, n_q_heads=2, n_kv_heads=2, seq_len=200)
    _compare(_run(case), _oracle(case))


def test_prefill_growing_logits_rescale():
    # keys grow along the sequence, so a row's running max climbs past the
    # lazy-rescale margin several times
    case = workloads.prefill_case(13, batch=1, n_q_heads=4, n_kv_heads=1, seq_len=900, key_ramp=6.0,
                                  tau_std=0.0, tau_bias=-1.0)
    _compare(_run(case), _oracle(case))


def test_prefill_non_finite_rows_past_the_end_are_never_used():
    # a cache with kv_stride > seq_len whose unused rows hold NaN
    case = workloads.prefill_case(14, batch=2, n_q_heads=4, n_kv_heads=2, seq_len=150, kv_stride=290,
                                  tail_fill=float("nan"))
    got = _run(case)
    assert np.isfinite(got["out"]).all() and np.isfinite(got["lse"]).all()
    _compare(got, _oracle(case))


def test_prefill_gate_at_one_half():
    case = workloads.prefill_case(15, batch=1, n_q_heads=2, n_kv_heads=1, seq_len=333, beta=0.0)
    got = _run(case)
    _compare(got, _oracle(case))
    np.testing.assert_allclose(got["gate_sum"][0, 0], (np.arange(333) + 1) / 2.0, rtol=1e-6)


def test_prefill_many_tiles():
    case = workloads.prefill_case(16, batch=1, n_q_heads=8, n_kv_heads=2, seq_len=2048)
    _compare(_run(case), _oracle(case))


def test_prefill_deterministic():
    case = workloads.prefill_case(17, batch=1, n_q_heads=4, n_kv_heads=1, seq_len=640)
    a, b = _run(case), _run(case)
    for n in ("out", "lse", "gate_sum"):
        np.testing.assert_array_equal(a[n], b[n])


def test_prefill_full_size_sampled_rows():
    """The shape the bench times (batch 1, 32 query / 8 KV heads, 8192 tokens,
    seed 0): sampled rows (the first and last rows of tiles, the sequence's
    ends, random interior rows) of sampled heads against the one-row oracle."""
    case = workloads.prefill_case(0, batch=1, n_q_heads=32, n_kv_heads=8, seq_len=8192)
    got = _run(case)
    G = case.n_q_heads // case.n_kv_heads
    rng = np.random.default_rng(1)
    rows = sorted({0, 1, 127, 128, 129, 4095, 4096, 8190, 8191, *rng.integers(0, 8192, 8).tolist()})
    for h in (0, 5, 17, 31):
        g = h // G
        q = case.q[0, h].float().double().numpy()
        tau = po.prefill_thresholds(q, case.tau_mode, case.w_tau[h], case.b_tau[h], None, case.offset_a)
        for i in rows:
            o, lse, r = po.prefill_row(q[i], case.k[0, g, :i + 1], case.v[0, g, :i + 1], tau[i], case.scale,
                                       case.beta)
            np.testing.assert_allclose(got["out"][0, h, i], o, rtol=OUT_RTOL, atol=OUT_ATOL, err_msg=f"{h} {i}")
            assert abs(got["lse"][0, h, i] - lse) <= LSE_ATOL, (h, i)
            assert abs(got["gate_sum"][0, h, i] - r) <= GATE_ATOL + GATE_RTOL * abs(r), (h, i)
