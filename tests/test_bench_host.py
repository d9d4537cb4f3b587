"""Host-side checks of the benchmark's accounting (no GPU): the algorithmic
byte counts, the whole-job aggregation, the max-over-ranks step time on a
2-rank gloo group, and the reference arm's rank-0-only output."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import workloads


def test_union_and_step_bytes_match_the_admitted_blocks():
    wl = workloads.custom(seed=5, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=64, block_size=16,
                          seq_lens=[250, 37], dtype=workloads.BF16, tau_bias=2.0, tau_std=1.0)
    r = oracle.decode(wl.q, wl.k, wl.v, wl.seq_lens, 16, "learned", wl.w_tau, wl.b_tau)
    ul = np.full((2, 2, wl.nb_max), -1)
    for i in range(2):
        for g in range(2):
            ids = np.flatnonzero(r["union"][i, g])
            ul[i, g, :len(ids)] = ids
    kv = bench.union_bytes(wl, ul, r["union_count"])
    expect = 0
    for i, T in enumerate(wl.seq_lens):
        for g in range(2):
            for blk in np.flatnonzero(r["union"][i, g]):
                expect += min(16, T - blk * 16) * 64 * 2 * 2
    assert kv == expect
    nb = wl.n_blocks(0) + wl.n_blocks(1)
    meta = nb * 2 * (4 * 64 + 4)
    qo = 2 * 2 * 8 * 64 * 2
    tau = 8 * (64 + 1) * 4
    assert bench.step_bytes(wl, kv) == kv + meta + qo + tau


def test_whole_job_value_is_weak_scaling_sum():
    assert bench.whole_job_gbs(1, 4_000_000_000, 1000.0) == pytest.approx(4.0)
    assert bench.whole_job_gbs(4, 4_000_000_000, 1000.0) == pytest.approx(16.0)
    assert bench.max_over_ranks(3.5, "cpu") == 3.5  # not distributed


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.0 + rank  # the slower rank decides
        out[rank] = bench.max_over_ranks(ms, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == 2.0 and out[1] == 2.0


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload, seed, steps, warmup = "c1_tiny", 0, 1, 0

    assert bench.run_reference(Args()) is None


def test_reference_arm_line_on_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class Args:
        workload, seed, steps, warmup = "c1_tiny", 0, 1, 0

    line = bench.run_reference(Args())
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
