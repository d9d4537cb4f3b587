"""Benchmark of the ETA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl eta|reference]

One step = one decode step (threshold + block screen, attention over the
admitted GQA-union blocks, split merge) over the whole batch of the workload,
launched as one replay of the step recorded into a CUDA graph
(eta_decode_graph_launch; --launch stream: one eta_decode call),
inputs resident in HBM, L2 flushed before every step outside the step's
events by reading a 256 MiB buffer (the evicted lines are clean, so the step
does not pay for writing back a flush buffer).  Prints ONE JSON line (rank 0).

value  = effective HBM bandwidth of the step: algorithmic bytes (K+V of the
         union-admitted blocks at their real lengths + all block metadata + q,
         threshold parameters and outputs) / device step time (mean of the K
         timed steps), summed over ranks (each rank decodes its own copy of
         the batch: weak scaling).  latency_us_distribution: a further run of
         max(100, K) steps (median, p10, p90).
e2e    = the same bytes / end-to-end step time through the public API with
         host buffers and a context that grows by one token per step (it
         crosses a block boundary inside the timed steps): one recorded graph
         per token (eta_step_graph_create) that copies the new lengths and
         positions up, appends the new K/V rows read by the append kernel from
         page-locked host memory (refreshing their block's metadata), decodes,
         and stores the output into page-locked host memory.
dense  = the same kernels with the screen off (every block loaded) on the
         same workload; configs = the other long-context workloads (default
         c3_long, c5_batched), screened and dense, each with its step time and
         fraction of the HBM peak.
roofline = the attention kernel: union K+V bytes per launch / its median
         isolated launch time (CUDA events on the launch stream between the
         library's kernels) vs the measured HBM copy bandwidth.
kernels_us = the isolated per-kernel times and how they add up to the step.
cpu_baseline = the CPU oracle (numpy, float64) on one KV head of sequence 0
         of the same workload, timed on this host's cores (median of 3, all
         cores and one core).
--impl reference runs that oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "decode-step latency (us) and effective HBM GB/s vs peak at 128K-512K ctx, 1 B200"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "c4_max"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ helpers

def _rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _workload_desc(wl):
    return (f"{wl.name}: batch {wl.batch}, {wl.n_q_heads} query / {wl.n_kv_heads} KV heads, d {wl.head_dim}, "
            f"ctx {min(wl.seq_lens)}-{max(wl.seq_lens)}, block {wl.block_size}, {wl.dtype}, {wl.tau_mode} tau")


def max_over_ranks(x: float, device) -> float:
    """Largest x over the ranks of the default process group (x itself when
    not distributed): the job's step time is the slowest rank's."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank_step: int, ms: float) -> float:
    """Aggregate effective bandwidth of all ranks (weak scaling: every rank
    moves the same bytes per step) for a max-over-ranks step time in ms."""
    return world * bytes_per_rank_step / (ms * 1e-3) / 1e9


def union_bytes(wl, union_list, union_count):
    """K+V bytes of the union-admitted blocks, tails at their real length."""
    tot = 0
    row = wl.head_dim * wl.elt_bytes
    for i, T in enumerate(wl.seq_lens):
        for g in range(wl.n_kv_heads):
            n = int(union_count[i, g])
            ids = union_list[i, g, :n].astype(np.int64)
            rows = np.minimum(wl.block_size, T - ids * wl.block_size)
            tot += int(rows.sum()) * row * 2
    return tot


def meta_record_bytes(head_dim, meta="fp16"):
    """Bytes of one block's metadata per KV head: fp16 centroid and spread +
    fp32 M, or e4m3 codes + two fp32 scales + fp32 M."""
    if meta == "box":
        return 4 * head_dim  # fp16 minima and maxima
    return 2 * head_dim + 12 if meta == "fp8" else 4 * head_dim + 4


def step_bytes(wl, kv_union, meta="fp16"):
    nb_total = sum(wl.n_blocks(i) for i in range(wl.batch)) * wl.n_kv_heads
    meta = nb_total * meta_record_bytes(wl.head_dim, meta)
    qo = 2 * wl.batch * wl.n_q_heads * wl.head_dim * wl.elt_bytes
    tau = wl.n_q_heads * (wl.head_dim + 1) * 4 if wl.tau_mode == "learned" else wl.n_q_heads * 4
    return kv_union + meta + qo + tau


class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "samples": len(sms)}


ATTEND_SOURCES = ("attend_tc.cu", "attend_common.cuh", "tc_common.cuh", "eta_device.cuh", "eta_internal.h")


def attend_source_sha1():
    """Hash of the sources the attention kernel is compiled from."""
    h = hashlib.sha1()
    for name in ATTEND_SOURCES:
        with open(os.path.join(ROOT, "learned_threshold_sparse_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic(workload):
    """dram bytes per attention launch from the committed ncu summary, or None
    when the attention kernel's sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(workload)
    if not ent or ent.get("source_sha1") != attend_source_sha1():
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ eta arm

KERNELS_PER_STEP = 3  # screen, attention, merge (the library's launches per decode step)


class Flush:
    """Evicts L2 before a step: reads a 256 MiB buffer (the evicted lines are
    clean, so the next step does not pay for writing back a flush buffer)."""

    def __init__(self, dev):
        self.buf = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        torch.sum(self.buf, dim=0, out=self.sink)


class Decode:
    """One workload resident on the device with its metadata, the decode
    parameters, a workspace, and (launch=graph) the step recorded as a CUDA
    graph; `dense` turns the screen off (every block loaded)."""

    def __init__(self, eta, wl, dev, args, dense=False):
        self.eta, self.wl, self.dense = eta, wl, dense
        self.q = wl.q.to(dev)
        self.k = wl.k.to(dev)
        self.v = wl.v.to(dev)
        self.seq = torch.tensor(wl.seq_lens, dtype=torch.int32, device=dev)
        self.w_tau = None if wl.w_tau is None else torch.from_numpy(wl.w_tau).to(dev)
        self.b_tau = None if wl.b_tau is None else torch.from_numpy(wl.b_tau).to(dev)
        self.c_tau = None if wl.c_tau is None else torch.from_numpy(wl.c_tau).to(dev)
        self.summ = eta.alloc_summary(wl.batch, wl.n_kv_heads, wl.max_ctx, wl.head_dim, wl.block_size, dev,
                                      fmt=args.meta)
        first = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
        eta.eta_block_summary_update(self.k, self.v, self.seq, self.summ, wl.block_size, first, wl.nb_max,
                                     wl.n_q_heads)
        self.kw = dict(w_tau=self.w_tau, b_tau=self.b_tau, c_tau=self.c_tau, scale=wl.scale, beta=wl.beta,
                       offset_a=wl.offset_a, z=wl.z, n_local_blocks=wl.n_local_blocks, screen_enabled=not dense,
                       attend_impl=args.attend_impl)
        # the admitted selection once, outside any timing, for the byte count
        sel = eta.decode(self.q, self.k, self.v, self.seq, self.summ, wl.block_size, wl.tau_mode, selection=True,
                         **self.kw)
        torch.cuda.synchronize()
        assert eta.eta_read_device_status(sel["workspace"]) == eta.ETA_OK
        uc = sel["union_count"].cpu().numpy()
        self.kv_union = union_bytes(wl, sel["union_list"].cpu().numpy(), uc)
        self.nbytes = step_bytes(wl, self.kv_union, args.meta)
        nb_total = sum(wl.n_blocks(i) for i in range(wl.batch)) * wl.n_kv_heads
        self.union_density = float(uc.sum()) / nb_total
        self.head_density = float(sel["admitted_count"].cpu().numpy().sum()) / (nb_total * wl.group)
        del sel
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((wl.batch, wl.n_q_heads), dtype=torch.float32, device=dev)
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for e in self.ev:  # materialise the cudaEvent_t handles the library records into
            e.record()
        torch.cuda.synchronize()
        self.params_ev = self.make_params(events=self.ev)
        self.params = self.make_params()
        self.trace = torch.zeros(eta.ETA_TRACE_SLOTS, dtype=torch.int64, device=dev)
        self.params_tr = self.make_params(trace=self.trace)
        self.ws = eta.alloc_workspace(eta.eta_decode_workspace_size(self.params), dev)
        for p in (self.params, self.params_ev, self.params_tr):
            p.workspace, p.workspace_bytes = self.ws.data_ptr(), self.ws.numel()
        self.graph = self.graph_tr = None
        if args.launch == "graph":
            keep = [self.q, self.k, self.v, self.seq, self.summ, self.out, self.lse, self.ws]
            self.graph = eta.DecodeGraph(self.params, keep)
            self.graph_tr = eta.DecodeGraph(self.params_tr, keep + [self.trace])

    def make_params(self, q=None, seq=None, out=None, events=None, trace=None):
        return self.eta.make_params(self.q if q is None else q, self.k, self.v, self.seq if seq is None else seq,
                                    self.summ, self.wl.block_size, self.wl.tau_mode,
                                    out=self.out if out is None else out, lse=self.lse, events=events, trace=trace,
                                    **self.kw)

    def step(self, stream):
        if self.graph is not None:
            self.graph.launch(stream)
        else:
            self.eta.eta_decode(self.params, stream)

    def step_traced(self, stream):
        if self.graph_tr is not None:
            self.graph_tr.launch(stream)
        else:
            self.eta.eta_decode(self.params_tr, stream)

    def close(self):
        for gname in ("graph", "graph_tr"):
            g = getattr(self, gname)
            if g is not None:
                g.close()
                setattr(self, gname, None)


def time_steps(fn, n, flush, stream):
    """n steps, each bracketed by events on the launch stream with an L2
    flush before it (outside the events); per-step milliseconds."""
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for _ in range(n):
        flush()
        s0.record(stream)
        fn()
        s1.record(stream)
        s1.synchronize()
        ms.append(s0.elapsed_time(s1))
    return ms


def kernel_times(d, n, flush, stream):
    """Per-kernel milliseconds from events the library records between its
    launches (screen, attention, merge), over n steps."""
    out = {"screen": [], "attend": [], "merge": []}
    for _ in range(n):
        flush()
        d.eta.eta_decode(d.params_ev, stream)
        d.ev[3].synchronize()
        out["screen"].append(d.ev[0].elapsed_time(d.ev[1]))
        out["attend"].append(d.ev[1].elapsed_time(d.ev[2]))
        out["merge"].append(d.ev[2].elapsed_time(d.ev[3]))
    return {k: statistics.median(v) for k, v in out.items()}


def step_breakdown(d, n, flush, stream):
    """Where one step's time goes: n steps launched the same way as the timed
    ones but with the library's step trace on (first-CTA start and last-CTA
    end of each kernel on the GPU's nanosecond timer, include/eta.h).  Per
    step, the parts below sum to the step's event time; medians are reported
    (so the medians need not sum exactly).  `outside` is the time of the step
    outside the kernels: the first kernel's launch and the last one's
    completion as the events see them."""
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    parts = {}
    for _ in range(n):
        flush()
        d.trace.zero_()
        s0.record(stream)
        d.step_traced(stream)
        s1.record(stream)
        s1.synchronize()
        step = s0.elapsed_time(s1) * 1e3
        tt = d.eta.trace_times(d.trace)
        us = lambda a, b: (tt[b] - tt[a]) / 1e3  # noqa: E731
        if "fused_first" in tt:
            p = {"start_to_first_tile": us("fused_first", "tile_first") if "tile_first" in tt else 0.0}
            p["tiles_to_end"] = us("tile_first" if "tile_first" in tt else "fused_first", "fused_last")
            span = us("fused_first", "fused_last")
        else:
            end = "merge_last" if tt.get("merge_last", 0) > tt["attend_last"] else "attend_last"
            p = {"screen": us("screen_first", "screen_last")}
            first = "tile_first" if "tile_first" in tt else "attend_first"
            p["screen_end_to_first_tile"] = us("screen_last", first)
            p["first_tile_to_attend_end"] = us(first, "attend_last")
            p["merge_tail"] = us("attend_last", end)
            span = us("screen_first", end)
        p["outside_kernels"] = step - span
        p["step"] = step
        for k, v in p.items():
            parts.setdefault(k, []).append(v)
    return {k: round(statistics.median(v), 2) for k, v in parts.items()}


def _pct(xs, p):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, max(0, int(round(p / 100.0 * (len(xs) - 1)))))]


def measure_config(d, args, flush, stream, peak):
    """Graph-replay step time (W warm-up, then max(100, K) steps) and the
    attention kernel's own time for one resident workload: the figures of a
    `configs` / `dense` entry."""
    for _ in range(args.warmup):
        flush()
        d.step(stream)
    torch.cuda.synchronize()
    ms = time_steps(lambda: d.step(stream), max(100, args.steps), flush, stream)
    kt = kernel_times(d, max(20, args.steps), flush, stream)
    med = statistics.median(ms)
    return {
        "workload": _workload_desc(d.wl),
        "screen": "off (dense)" if d.dense else "on",
        "steps": len(ms),
        "step_us_median": round(med * 1e3, 2),
        "step_us_mean": round(statistics.mean(ms) * 1e3, 2),
        "step_us_p10_p90": [round(_pct(ms, 10) * 1e3, 2), round(_pct(ms, 90) * 1e3, 2)],
        "bytes_per_step": d.nbytes,
        "kv_union_bytes_per_step": d.kv_union,
        "union_density": round(d.union_density, 4),
        "head_density": round(d.head_density, 4),
        "step_gbs": round(d.nbytes / (med * 1e-3) / 1e9, 1),
        "step_frac_of_peak": round(d.nbytes / (med * 1e-3) / 1e9 / peak, 4),
        "attend_us_isolated": round(kt["attend"] * 1e3, 2),
        "attend_frac_of_peak": round(d.kv_union / (kt["attend"] * 1e-3) / 1e9 / peak, 4),
        "breakdown_us": step_breakdown(d, 50, flush, stream),
    }


def append_time(eta, d, flush, stream, n=100):
    """One-token append timed alone (eta_append_kv: write the token's K/V rows
    of every (sequence, KV head) and re-summarise the block holding it), the
    L2 flushed before each; the token re-written is the last one of each
    sequence with its own values, so the cache is unchanged.  Median us."""
    wl = d.wl
    last = [max(0, T - 1) for T in wl.seq_lens]
    k_new = torch.stack([d.k[i, :, t] for i, t in enumerate(last)]).contiguous()
    v_new = torch.stack([d.v[i, :, t] for i, t in enumerate(last)]).contiguous()
    pos = torch.tensor(last, dtype=torch.int32, device=d.q.device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for _ in range(n):
        flush()
        e0.record(stream)
        eta.eta_append_kv(d.k, d.v, d.seq, d.summ, wl.block_size, k_new, v_new, pos, wl.n_q_heads, stream=stream)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    return round(statistics.median(ms) * 1e3, 2)


def e2e_append(eta, d, args, flush, stream, dev):
    """End to end through the public API with host buffers, the sequence
    growing by one token per step: each step's new query, key and value rows
    are written into page-locked host memory, the new lengths and positions
    are copied up (a copy kernel reading the page-locked buffer), the append
    kernel reads the rows from host memory, writes them into the cache and
    refreshes their block's metadata, the decode runs and stores its output
    into page-locked host memory; one recorded graph per step
    (eta_step_graph_create).  The context starts b + K/2 tokens short of the
    workload's so that appends cross a block boundary inside the timed
    steps; the appended rows are the workload's own rows at those positions,
    so the cache ends as it began.  Returns (per-step ms, h2d bytes, d2h bytes,
    note)."""
    wl = d.wl
    B, Hq, Hkv, hd, b = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.block_size
    K = args.steps
    T0 = [max(1, min(T - b - K // 2, wl.max_ctx - K)) for T in wl.seq_lens]
    nq, nkv = B * Hq * hd, B * Hkv * hd
    rows_h = torch.empty(nq + 2 * nkv, dtype=wl.q.dtype).pin_memory()
    rows_h[:nq].copy_(wl.q.reshape(-1))
    lens_h = torch.zeros(2 * B, dtype=torch.int32).pin_memory()
    lens_d = torch.zeros(2 * B, dtype=torch.int32, device=dev)
    seq_d, pos_d = lens_d[:B], lens_d[B:]
    q_in = torch.empty_like(d.q)
    out_h = torch.empty_like(wl.q).pin_memory()
    p = d.make_params(q=q_in, seq=seq_d, out=out_h)
    p.workspace, p.workspace_bytes = d.ws.data_ptr(), d.ws.numel()
    g = eta.StepGraph(p, k_new=rows_h[nq:nq + nkv].view(B, Hkv, hd), v_new=rows_h[nq + nkv:].view(B, Hkv, hd),
                      positions=pos_d, q_new=rows_h[:nq].view(B, Hq, hd), h2d=lens_h, h2d_dst=lens_d,
                      tensors=[q_in, d.k, d.v, d.summ, d.lse, d.ws, out_h, lens_d])
    k_rows = rows_h[nq:nq + nkv].view(B, Hkv, hd)
    v_rows = rows_h[nq + nkv:].view(B, Hkv, hd)

    def reset():
        # outside the events: lengths back to T0 and the block holding token
        # T0 - 1 summarised over its tokens < T0 again
        seq_d.copy_(torch.tensor(T0, dtype=torch.int32))
        first = torch.tensor([t - 1 for t in T0], dtype=torch.int32, device=dev)
        eta.eta_block_summary_update(d.k, d.v, seq_d, d.summ, b, first, 1, Hq)
        torch.cuda.synchronize()

    def host_token(s):
        for i in range(B):
            pos = T0[i] + s
            k_rows[i].copy_(wl.k[i, :, pos])
            v_rows[i].copy_(wl.v[i, :, pos])
            lens_h[i] = pos + 1
            lens_h[B + i] = pos

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    try:
        for phase, n in (("warmup", args.warmup), ("timed", K)):
            reset()
            for s in range(n):
                host_token(s)
                flush()
                e0.record(stream)
                g.launch(stream)
                e1.record(stream)
                e1.synchronize()
                if phase == "timed":
                    ms.append(e0.elapsed_time(e1))
        # the output of the last token equals a fresh decode of the state it left
        check = torch.empty_like(d.q)
        pc = d.make_params(q=q_in, seq=seq_d, out=check)
        pc.workspace, pc.workspace_bytes = d.ws.data_ptr(), d.ws.numel()
        eta.eta_decode(pc, stream)
        torch.cuda.synchronize()
        assert eta.eta_read_device_status(d.ws) == eta.ETA_OK
        assert torch.equal(check.cpu(), out_h), "e2e output differs from a decode of the final state"
        crossed = any(T0[i] // b != (T0[i] + K - 1) // b for i in range(B))
        # the same token path recorded with the step trace on: where its time goes
        pt = d.make_params(q=q_in, seq=seq_d, out=out_h, trace=d.trace)
        pt.workspace, pt.workspace_bytes = d.ws.data_ptr(), d.ws.numel()
        gt = eta.StepGraph(pt, k_new=rows_h[nq:nq + nkv].view(B, Hkv, hd), v_new=rows_h[nq + nkv:].view(B, Hkv, hd),
                           positions=pos_d, q_new=rows_h[:nq].view(B, Hq, hd), h2d=lens_h, h2d_dst=lens_d,
                           tensors=[q_in, d.k, d.v, d.summ, d.lse, d.ws, out_h, lens_d, d.trace])
        try:
            reset()
            order = ["in_first", "in_last", "append_first", "append_last", "screen_first", "screen_last",
                     "tile_first", "attend_last", "merge_last", "out_first", "out_last"]
            parts = {}
            for s in range(min(K, 30)):
                host_token(s)
                flush()
                d.trace.zero_()
                e0.record(stream)
                gt.launch(stream)
                e1.record(stream)
                e1.synchronize()
                tt = eta.trace_times(d.trace)
                seq_t = [(n, tt[n]) for n in order if n in tt]
                for (a, ta), (bn, tb) in zip(seq_t, seq_t[1:]):
                    parts.setdefault(f"{a}->{bn}", []).append((tb - ta) / 1e3)
                parts.setdefault("outside_kernels", []).append(e0.elapsed_time(e1) * 1e3 - (seq_t[-1][1] - seq_t[0][1]) / 1e3)
                parts.setdefault("step", []).append(e0.elapsed_time(e1) * 1e3)
            e2e_bd = {k: round(statistics.median(v), 2) for k, v in parts.items()}
        finally:
            gt.close()
    finally:
        g.close()
        # back to the workload's own lengths and tail metadata
        d.seq.copy_(torch.tensor(wl.seq_lens, dtype=torch.int32))
        first = torch.tensor([max(0, T - 1) for T in wl.seq_lens], dtype=torch.int32, device=dev)
        eta.eta_block_summary_update(d.k, d.v, d.seq, d.summ, b, first, 1, Hq)
        torch.cuda.synchronize()
    h2d = rows_h.numel() * rows_h.element_size() + lens_h.numel() * 4
    d2h = out_h.numel() * out_h.element_size()
    note = (f"context grows one token per step from {min(T0)} (seq 0: {T0[0]} -> {T0[0] + K}); appends cross a "
            f"block boundary inside the timed steps: {crossed}; bytes per step counted at the full context")
    return ms, h2d, d2h, note, e2e_bd


def run_eta(args):
    import learned_threshold_sparse_b200 as eta

    rank, local_rank, world = _rank_env()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = Flush(dev)
    peak, peak_kind = _peaks()

    wl = workloads.make(args.workload, args.seed)
    d = Decode(eta, wl, dev, args, dense=args.dense)
    for _ in range(args.warmup):
        flush()
        d.step(stream)
    torch.cuda.synchronize()

    # Timed region: exactly K steps, each bracketed by events on the launch
    # stream; the L2 flush before every step stays outside the events.  The
    # clock sampler runs over this and every later measurement.
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    step_ms = time_steps(lambda: d.step(stream), args.steps, flush, stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    wall_s = time.perf_counter() - t_wall
    ms = max_over_ranks(statistics.mean(step_ms), dev)
    value = whole_job_gbs(world, d.nbytes, ms)
    # A longer run of the same step for the distribution (median of >= 100).
    dist_ms = time_steps(lambda: d.step(stream), max(100, args.steps), flush, stream)
    kt = kernel_times(d, max(20, args.steps), flush, stream)
    bd = step_breakdown(d, 50, flush, stream)
    app_us = append_time(eta, d, flush, stream)
    assert eta.eta_read_device_status(d.ws) == eta.ETA_OK
    med = statistics.median(dist_ms)

    # ---- end to end through the public API, host buffers, growing context
    e2e_ms, h2d, d2h, e2e_note, e2e_bd = e2e_append(eta, d, args, flush, stream, dev)
    e2e = max_over_ranks(statistics.mean(e2e_ms), dev)
    d.close()
    main = dict(kv_union=d.kv_union, nbytes=d.nbytes, union_density=d.union_density, head_density=d.head_density)
    del d
    torch.cuda.empty_cache()

    # ---- the dense path of the same kernels, and the other long-context configs
    extra = {}
    if world == 1 and not args.no_configs:
        if not args.dense:
            dd = Decode(eta, wl, dev, args, dense=True)
            extra["dense"] = measure_config(dd, args, flush, stream, peak)
            dd.close()
            del dd
            torch.cuda.empty_cache()
        cfgs = {}
        for name in [c for c in args.configs.split(",") if c and c != args.workload]:
            w2 = workloads.make(name, args.seed)
            entry = {}
            for dense in (False, True):
                x = Decode(eta, w2, dev, args, dense=dense)
                entry["dense" if dense else "screened"] = measure_config(x, args, flush, stream, peak)
                x.close()
                del x
                torch.cuda.empty_cache()
            cfgs[name] = entry
            del w2
        extra["configs"] = cfgs
        if args.attend_impl == 0 and not args.dense:
            # the single-launch alternative (ETA_ATTEND_FUSED: screen, attention
            # and merge in one persistent kernel) on the same workloads
            fa = argparse.Namespace(**vars(args))
            fa.attend_impl = 3
            fused = {}
            for name in [args.workload] + [c for c in args.configs.split(",") if c and c != args.workload]:
                w2 = workloads.make(name, args.seed)
                x = Decode(eta, w2, dev, fa)
                fused[name] = measure_config(x, fa, flush, stream, peak)
                x.close()
                del x, w2
                torch.cuda.empty_cache()
            extra["fused_kernel"] = {"note": ("attend_impl = ETA_ATTEND_FUSED: one launch per step (screen, "
                                              "attention, merge); attend_us_isolated is that launch"), **fused}
    clk = clocks.stop()
    if world == 1 and not args.no_configs and not args.dense:
        # the causal forward pass (prefill) at its default shape on the same
        # GPU, after the decode's clock record: its own line's figures
        pa = argparse.Namespace(**vars(args))
        pa.steps = 20
        pl = run_prefill(pa)
        extra["prefill"] = {"workload": pl["config"]["workload"], "metric": pl["metric"],
                            **{k: pl[k] for k in ("value", "unit", "statistic", "ms_per_step", "ms_mean", "tflops_mean",
                                                  "ms_p10_p90", "roofline", "clocks")}}
        torch.cuda.empty_cache()

    att = kt["attend"]
    achieved = main["kv_union"] / (att * 1e-3) / 1e9
    traffic = _traffic(args.workload + ("_dense" if args.dense else ""))
    line = None
    if rank == 0:
        cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline(wl, args)
        iso = {k: round(v * 1e3, 2) for k, v in kt.items()}
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms, 6),
            "latency_us": round(ms * 1e3, 2),
            "latency_us_median": round(statistics.median(step_ms) * 1e3, 2),
            "latency_us_distribution": {"steps": len(dist_ms), "median": round(med * 1e3, 2),
                                        "mean": round(statistics.mean(dist_ms) * 1e3, 2),
                                        "p10": round(_pct(dist_ms, 10) * 1e3, 2),
                                        "p90": round(_pct(dist_ms, 90) * 1e3, 2),
                                        "note": "a second run of the same step after the K timed steps"},
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": wl.dtype,
            "accum": "f32",
            "data": "synthetic",
            "config": {
                "workload": _workload_desc(wl),
                "seed": args.seed,
                "screen": "off (dense)" if args.dense else "on",
                "metadata": args.meta,
                "attend_impl": {0: "auto", 1: "simt", 2: "tc", 3: "fused"}[args.attend_impl],
                "union_density": round(main["union_density"], 4),
                "head_density": round(main["head_density"], 4),
                "bytes_per_step": main["nbytes"],
                "kv_union_bytes_per_step": main["kv_union"],
                "l2": "flushed before every step by reading a 256 MiB buffer (outside the step events)",
                "launch": ("one CUDA graph replay per step (eta_decode_graph_launch)" if args.launch == "graph"
                           else "stream launches (eta_decode)"),
                "parallelism": f"replicas x{world} (each rank decodes its own batch)",
            },
            "kernels_us": {
                "isolated": iso,
                "sum_isolated": round(sum(iso.values()), 2),
                "step_median": round(med * 1e3, 2),
                "overlap_and_gaps": round(med * 1e3 - sum(iso.values()), 2),
                "note": ("medians of a run with library events recorded between the kernels; those events stop "
                         "the kernels' programmatic-launch overlap and add a launch gap to each, so the isolated "
                         "times sum to more than the step: step = sum_isolated + overlap_and_gaps; "
                         "breakdown_us decomposes the step itself"),
            },
            "breakdown_us": {**bd, "note": ("medians over 50 graph replays with the library's step trace on: "
                                            "per step the parts sum to the step's event time")},
            "append_us": {"median": app_us, "steps": 100,
                          "note": ("eta_append_kv of one token per sequence (K/V rows written, their block "
                                   "re-summarised), timed alone with the L2 flushed; not part of a decode step")},
            "roofline": {"kernel": "attend", "bound": "hbm", "achieved": round(achieved, 2),
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": main["kv_union"],
                         "time": "isolated attention-kernel time (events on the launch stream; includes its launch gap)"},
            "step_frac_of_peak": round(main["nbytes"] / (ms * 1e-3) / 1e9 / peak, 4),
            "e2e": {"value": round(whole_job_gbs(world, main["nbytes"], e2e), 2), "unit": UNIT,
                    "ms_per_step": round(e2e, 6), "us_median": round(statistics.median(e2e_ms) * 1e3, 2),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "io": ("one graph per token (eta_step_graph_create): new lengths and positions copied up by a "
                           "kernel reading page-locked memory, the append kernel reads the new q, k, v rows from "
                           "page-locked host memory, the decode stores out into page-locked host memory"),
                    "mode": e2e_note,
                    "breakdown_us": {**e2e_bd, "note": ("medians over 30 tokens of the same graph recorded with the "
                                                        "step trace on: intervals between consecutive kernel "
                                                        "first-starts / last-ends, in step order, plus the time "
                                                        "outside the kernels; per token they sum to the step")}},
            **extra,
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "clocks": clk,
            "wall_s_timed_region": round(wall_s, 3),
            "cpu_baseline": cpu,
        }
    if world > 1:
        torch.distributed.destroy_process_group()
    return line


# ------------------------------------------------------------------ oracle arm

def _oracle_sample(wl):
    """One KV head (with its G query heads) of sequence 0: the bounded sample
    the CPU oracle is timed on."""
    G = wl.group
    return wl.with_params(batch=1, n_q_heads=G, n_kv_heads=1, seq_lens=[wl.seq_lens[0]],
                          q=wl.q[:1, :G].contiguous(), k=wl.k[:1, :1], v=wl.v[:1, :1],
                          w_tau=None if wl.w_tau is None else wl.w_tau[:G],
                          b_tau=None if wl.b_tau is None else wl.b_tau[:G],
                          c_tau=None if wl.c_tau is None else wl.c_tau[:G])


def _oracle_step(oracle, s, summary):
    return oracle.decode(s.q, s.k, s.v, s.seq_lens, s.block_size, s.tau_mode, w_tau=s.w_tau, b_tau=s.b_tau,
                         c_tau=s.c_tau, scale=s.scale, beta=s.beta, offset_a=s.offset_a, z=s.z,
                         n_local_blocks=s.n_local_blocks, screen_enabled=s.screen_enabled, summary=summary)


def _sample_bytes(s, r):
    ul = np.full((1, 1, s.nb_max), -1, np.int64)
    ids = np.flatnonzero(r["union"][0, 0])
    ul[0, 0, :len(ids)] = ids
    return step_bytes(s, union_bytes(s, ul, np.array([[len(ids)]])))


def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(wl, args, repeats=3):
    """The CPU oracle (numpy, float64) on a bounded sample of the workload:
    sequence 0, KV head 0 with its G query heads (1 / (batch x KV heads) of
    the step), block metadata computed once beforehand.  Median of `repeats`
    runs with numpy's thread pools limited to all host cores, and again to one
    core.  value = the sample's algorithmic bytes / median seconds."""
    import oracle
    from threadpoolctl import threadpool_limits

    s = _oracle_sample(wl)
    summary = oracle.summarize(s.k, s.seq_lens, s.block_size)
    cores = _host_cores()
    med = {}
    r = None
    for label, n in (("all", cores), ("one", 1)):
        with threadpool_limits(limits=n):
            ts = []
            for _ in range(repeats):
                t0 = time.perf_counter()
                r = _oracle_step(oracle, s, summary)
                ts.append(time.perf_counter() - t0)
        med[label] = statistics.median(ts)
    nbytes = _sample_bytes(s, r)
    per_step = wl.batch * wl.n_kv_heads
    return {"value": round(nbytes / med["all"] / 1e9, 4), "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "repeats": repeats, "statistic": "median",
            "seconds_per_sample": round(med["all"], 4),
            "seconds_per_sample_one_core": round(med["one"], 4),
            "value_one_core": round(nbytes / med["one"] / 1e9, 4),
            "samples_per_step": per_step,
            "seconds_per_step_estimated": round(med["all"] * per_step, 3),
            "sample": (f"{wl.name} seed {wl.seed}: sequence 0, KV head 0 with its {s.n_q_heads} query heads "
                       f"(1/{per_step} of the step), block metadata precomputed; numpy float64; 'cores' = the "
                       "thread limit given to numpy's pools (its matrix products use them, its elementwise work "
                       "runs on one thread)")}


def run_reference(args):
    rank, _, world = _rank_env()
    if rank != 0:
        return None
    import oracle

    wl = workloads.make(args.workload, args.seed)
    s = _oracle_sample(wl)
    summary = oracle.summarize(s.k, s.seq_lens, s.block_size)
    for _ in range(args.warmup):
        _oracle_step(oracle, s, summary)
    ts = []
    r = None
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = _oracle_step(oracle, s, summary)
        ts.append(time.perf_counter() - t0)
    sec = statistics.mean(ts)
    nbytes = _sample_bytes(s, r)
    value = round(nbytes / sec / 1e9, 4)
    cores = _host_cores()
    sample = (f"{wl.name} seed {wl.seed}: each step is sequence 0, KV head 0 with its {s.n_q_heads} query heads "
              f"(1/{wl.batch * wl.n_kv_heads} of the decode step), block metadata precomputed; numpy float64")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "seed": args.seed, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_prefill(args):
    """Causal forward pass (eta_prefill) over a whole sequence: tensor flops of
    the two contractions over the causal triangle per second, against the
    measured dense bf16 peak (median step; the mean beside it).  Not the
    decode metric; printed on its own line."""
    import learned_threshold_sparse_b200 as eta

    B, Hq, Hkv, T = (int(x) for x in args.prefill_shape.split(","))
    d = 128
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    case = workloads.prefill_case(args.seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv, seq_len=T, head_dim=d)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    w = torch.from_numpy(case.w_tau).to(dev)
    bt = torch.from_numpy(case.b_tau).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    gate = torch.empty_like(lse)
    ws = eta.alloc_workspace(eta.PREFILL_WORKSPACE_BYTES, dev)
    params = eta.make_prefill_params(q, k, v, T, case.tau_mode, w_tau=w, b_tau=bt, scale=case.scale,
                                     beta=case.beta, offset_a=case.offset_a, out=out, lse=lse, gate_sum=gate,
                                     workspace=ws)
    stream = torch.cuda.current_stream(dev)
    flush_buf = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        eta.eta_prefill(params, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    ms = []
    steps = max(args.steps, 20)
    for _ in range(steps):
        torch.sum(flush_buf, dim=0, out=flush_sink)
        e0.record(stream)
        eta.eta_prefill(params, stream)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    clk = clocks.stop()
    assert eta.eta_read_device_status(ws) == eta.ETA_OK
    flops = 4.0 * d * (T * (T + 1) / 2) * B * Hq
    t = statistics.median(ms)
    tflops = flops / (t * 1e-3) / 1e12
    t_mean = statistics.mean(ms)
    peak_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak, kind = 1590.0, "fallback"
    if os.path.exists(peak_path):
        with open(peak_path) as f:
            peak, kind = float(json.load(f)["bf16_tflops"]), "measured"
    return {
        "metric": "ETA causal forward (prefill) tensor TFLOP/s",
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": round(t, 4),
        "statistic": "median of the timed steps",
        "ms_mean": round(t_mean, 4),
        "tflops_mean": round(flops / (t_mean * 1e-3) / 1e12, 2),
        "ms_p10_p90": [round(_pct(ms, 10), 4), round(_pct(ms, 90), 4)],
        "higher_is_better": True,
        "dtype": "bf16",
        "accum": "f32",
        "data": "synthetic",
        "config": {"workload": f"prefill: batch {B}, {Hq} query / {Hkv} KV heads, seq {T}, d {d}, bf16, learned tau",
                   "flops_per_step": flops,
                   "l2": "flushed before every step by reading a 256 MiB buffer (outside the events)"},
        "roofline": {"kernel": "prefill_tc", "bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                     "peak_kind": kind + " dense bf16 (burst)", "unit": "TFLOP/s", "frac": round(tflops / peak, 4)},
        "gpu_launches": steps,
        "clocks": clk,
    }


def run_calibrate(args):
    """Offline calibration histogram (eta_calibration_histogram) over a batch of
    calibration sequences: causal logits binned per second, and the time of one
    full pass; the constants solved from it on the host."""
    import learned_threshold_sparse_b200 as eta

    B, Hq, Hkv, T = (int(x) for x in args.calib_shape.split(","))
    d = 128
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    case = workloads.prefill_case(args.seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv, seq_len=T, head_dim=d)
    q, k = case.q.to(dev), case.k.to(dev)
    hist = torch.zeros((Hq, 4096 + 2), dtype=torch.float64, device=dev)
    for _ in range(args.warmup):
        eta.calibration_histogram(q, k, T, scale=case.scale, hist=hist)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for _ in range(args.steps):
        hist.zero_()
        e0.record()
        eta.calibration_histogram(q, k, T, scale=case.scale, hist=hist)
        e1.record()
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    c = eta.calibrate_constants(hist, -8.0, 8.0, 0.38)
    t = statistics.mean(ms)
    pairs = B * Hq * T * (T + 1) / 2
    return {
        "metric": "ETA offline calibration: causal logits binned per second",
        "value": round(pairs / (t * 1e-3) / 1e9, 3),
        "unit": "Glogits/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t, 4),
        "higher_is_better": True,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"calibration: {B} sequences, {Hq} query / {Hkv} KV heads, seq {T}, d {d}, bf16, "
                               "4096 bins over [-8, 8)",
                   "tensor_flops_equivalent_per_step": 2.0 * d * pairs,
                   "constants_at_density_0.38": [round(float(x), 4) for x in c[:4]]},
        "gpu_launches": args.steps,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="eta", choices=["eta", "reference"])
    ap.add_argument("--attend-impl", type=int, default=0, choices=[0, 1, 2, 3])
    ap.add_argument("--dense", action="store_true", help="screen off: every block loaded")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="decode step as one recorded CUDA graph (default) or as stream launches")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default="c2_single,c3_long,c5_batched",
                    help="other workloads measured (screened and dense) after the main line")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the dense arm, the other workloads, the single-launch kernel and the prefill")
    ap.add_argument("--meta", default="fp16", choices=["fp16", "fp8", "box"],
                    help="block metadata format (box: the comparison coordinate-box screen)")
    ap.add_argument("--prefill", action="store_true", help="time the causal forward pass instead of the decode step")
    ap.add_argument("--prefill-shape", default="1,32,8,8192", help="batch,n_q_heads,n_kv_heads,seq_len")
    ap.add_argument("--calibrate", action="store_true", help="time the offline calibration histogram")
    ap.add_argument("--calib-shape", default="16,16,4,4096", help="sequences,n_q_heads,n_kv_heads,seq_len")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.prefill:
        line = run_prefill(args)
    elif args.calibrate:
        line = run_calibrate(args)
    else:
        line = run_reference(args) if args.impl == "reference" else run_eta(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
