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
         threshold parameters and outputs) / device step time, summed over
         ranks (each rank decodes its own copy of the batch: weak scaling).
e2e    = the same bytes / end-to-end step time through the public API: the
         new token's q, k, v copied in one transfer from pinned host memory,
         the append (K/V rows written, their block's metadata refreshed), the
         decode step, the output copied back to pinned host memory; by
         default one recorded graph (eta_step_graph_create) in which the
         append kernel reads the new rows from pinned host memory and the
         decode stores its output into pinned host memory directly; with
         --launch stream, separate calls with copy-engine transfers.
roofline = the attention kernel: union K+V bytes per launch / its mean
         launch time (CUDA events on the launch stream, second run of K
         steps) vs the measured HBM copy bandwidth.
cpu_baseline = the CPU oracle (numpy, fp64) on one KV head of the same
         workload, timed on this host.
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

    wl = workloads.make(args.workload, args.seed)
    q = wl.q.to(dev)
    k = wl.k.to(dev)
    v = wl.v.to(dev)
    seq = torch.tensor(wl.seq_lens, dtype=torch.int32, device=dev)
    w_tau = None if wl.w_tau is None else torch.from_numpy(wl.w_tau).to(dev)
    b_tau = None if wl.b_tau is None else torch.from_numpy(wl.b_tau).to(dev)
    c_tau = None if wl.c_tau is None else torch.from_numpy(wl.c_tau).to(dev)
    summ = eta.alloc_summary(wl.batch, wl.n_kv_heads, wl.max_ctx, wl.head_dim, wl.block_size, dev, fmt=args.meta)
    first = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
    eta.eta_block_summary_update(k, v, seq, summ, wl.block_size, first, wl.nb_max, wl.n_q_heads)

    # selection once (outside timing) for the byte count
    sel = eta.decode(q, k, v, seq, summ, wl.block_size, wl.tau_mode, w_tau=w_tau, b_tau=b_tau, c_tau=c_tau,
                     scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
                     n_local_blocks=wl.n_local_blocks, screen_enabled=not args.dense,
                     attend_impl=args.attend_impl, selection=True)
    torch.cuda.synchronize()
    assert eta.eta_read_device_status(sel["workspace"]) == eta.ETA_OK
    uc = sel["union_count"].cpu().numpy()
    ul = sel["union_list"].cpu().numpy()
    kv_union = union_bytes(wl, ul, uc)
    nbytes = step_bytes(wl, kv_union, args.meta)
    nb_total = sum(wl.n_blocks(i) for i in range(wl.batch)) * wl.n_kv_heads
    union_density = float(uc.sum()) / nb_total
    head_density = float(sel["admitted_count"].cpu().numpy().sum()) / (nb_total * wl.group)

    out = torch.empty_like(q)
    lse = torch.empty((wl.batch, wl.n_q_heads), dtype=torch.float32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:  # materialise the cudaEvent_t handles the library records into
        e.record()
    torch.cuda.synchronize()
    params = eta.make_params(q, k, v, seq, summ, wl.block_size, wl.tau_mode, w_tau=w_tau, b_tau=b_tau,
                             c_tau=c_tau, scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
                             n_local_blocks=wl.n_local_blocks, screen_enabled=not args.dense,
                             attend_impl=args.attend_impl, out=out, lse=lse, events=ev)
    ws = eta.alloc_workspace(eta.eta_decode_workspace_size(params), dev)
    params.workspace = ws.data_ptr()
    params.workspace_bytes = ws.numel()
    stream = torch.cuda.current_stream(dev)
    flush_buf = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    class _Flush:
        @staticmethod
        def fill_(_):
            torch.sum(flush_buf, dim=0, out=flush_sink)

    flush = _Flush()

    def one_step():
        eta.eta_decode(params, stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        one_step()
    torch.cuda.synchronize()

    params_plain = eta.make_params(q, k, v, seq, summ, wl.block_size, wl.tau_mode, w_tau=w_tau, b_tau=b_tau,
                                   c_tau=c_tau, scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
                                   n_local_blocks=wl.n_local_blocks, screen_enabled=not args.dense,
                                   attend_impl=args.attend_impl, out=out, lse=lse)
    params_plain.workspace = ws.data_ptr()
    params_plain.workspace_bytes = ws.numel()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.launch == "graph":
        # the serving-loop launch path: the step recorded once, replayed per step
        graph = eta.DecodeGraph(params_plain, [q, k, v, seq, summ, out, lse, ws])

        def timed_step():
            graph.launch(stream)
    else:
        graph = None

        def timed_step():
            eta.eta_decode(params_plain, stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        timed_step()
    torch.cuda.synchronize()

    # Timed region: K steps, each bracketed by events on the launch stream;
    # the L2 flush before every step stays outside the events.
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    step_ms = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for _ in range(args.steps):
        flush.fill_(1.0)
        s0.record(stream)
        timed_step()
        s1.record(stream)
        s1.synchronize()
        step_ms.append(s0.elapsed_time(s1))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    wall_s = time.perf_counter() - t_wall
    # Per-kernel breakdown over a second run of K steps: the library records
    # events before the screen, before the attention kernel and after it.
    screen_ms, attend_ms, merge_ms = [], [], []
    for _ in range(args.steps):
        flush.fill_(1.0)
        one_step()
        ev[3].synchronize()
        screen_ms.append(ev[0].elapsed_time(ev[1]))
        attend_ms.append(ev[1].elapsed_time(ev[2]))
        merge_ms.append(ev[2].elapsed_time(ev[3]))
    clk = clocks.stop()
    assert eta.eta_read_device_status(ws) == eta.ETA_OK

    ms = max_over_ranks(statistics.mean(step_ms), dev)
    value = whole_job_gbs(world, nbytes, ms)

    # ---- end to end through the public API, host buffers: the step's new
    # query, key and value rows go up in one copy from pinned memory, the
    # append writes the K/V rows and refreshes their block, the decode runs,
    # the output comes back to pinned memory.
    B_, Hq_, Hkv_, d_ = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    nq, nkv = B_ * Hq_ * d_, B_ * Hkv_ * d_
    knew = torch.stack([wl.k[i, :, wl.seq_lens[i] - 1] for i in range(B_)])
    vnew = torch.stack([wl.v[i, :, wl.seq_lens[i] - 1] for i in range(B_)])
    packed_h = torch.cat([wl.q.reshape(-1), knew.reshape(-1), vnew.reshape(-1)]).pin_memory()
    packed_d = torch.empty(packed_h.shape, dtype=packed_h.dtype, device=dev)
    q_in = packed_d[:nq].view(B_, Hq_, d_)
    k_in = packed_d[nq:nq + nkv].view(B_, Hkv_, d_)
    v_in = packed_d[nq + nkv:].view(B_, Hkv_, d_)
    out_h = torch.empty_like(wl.q).pin_memory()
    last = torch.tensor([T - 1 for T in wl.seq_lens], dtype=torch.int32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    params_e2e = eta.make_params(q_in, k, v, seq, summ, wl.block_size, wl.tau_mode, w_tau=w_tau, b_tau=b_tau,
                                 c_tau=c_tau, scale=wl.scale, beta=wl.beta, offset_a=wl.offset_a, z=wl.z,
                                 n_local_blocks=wl.n_local_blocks, screen_enabled=not args.dense,
                                 attend_impl=args.attend_impl, out=out, lse=lse)
    params_e2e.workspace = ws.data_ptr()
    params_e2e.workspace_bytes = ws.numel()

    if args.launch == "graph":
        # the whole token as one recorded graph: the append kernel reads the
        # new q, k, v rows from page-locked host memory (and puts q where the
        # decode reads it), the decode stores its output straight into
        # page-locked host memory
        params_e2e.out = out_h.data_ptr()
        graph_e2e = eta.StepGraph(params_e2e, k_new=packed_h[nq:nq + nkv].view(B_, Hkv_, d_),
                                  v_new=packed_h[nq + nkv:].view(B_, Hkv_, d_), positions=last,
                                  q_new=packed_h[:nq].view(B_, Hq_, d_),
                                  tensors=[q_in, k, v, seq, summ, lse, ws, out_h])

        def e2e_step():
            graph_e2e.launch(stream)
    else:
        graph_e2e = None

        def e2e_step():
            packed_d.copy_(packed_h, non_blocking=True)
            eta.eta_append_kv(k, v, seq, summ, wl.block_size, k_in, v_in, last, wl.n_q_heads, stream)
            eta.eta_decode(params_e2e, stream)
            out_h.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    assert torch.equal(out_h, out.cpu())
    for g in (graph, graph_e2e):
        if g is not None:
            g.close()
    e2e = max_over_ranks(statistics.mean(e2e_ms), dev)
    h2d = packed_h.numel() * wl.elt_bytes
    d2h = out_h.numel() * wl.elt_bytes

    peak, peak_kind = _peaks()
    att_ms = statistics.mean(attend_ms)
    achieved = kv_union / (att_ms * 1e-3) / 1e9
    traffic = _traffic(args.workload + ("_dense" if args.dense else ""))

    line = None
    if rank == 0:
        cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline(wl, args)
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms, 6),
            "latency_us": round(ms * 1e3, 2),
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
                "attend_impl": {0: "auto", 1: "simt", 2: "tc"}[args.attend_impl],
                "union_density": round(union_density, 4),
                "head_density": round(head_density, 4),
                "bytes_per_step": nbytes,
                "kv_union_bytes_per_step": kv_union,
                "l2": "flushed before every step by reading a 256 MiB buffer (outside the step events)",
                "launch": ("one CUDA graph replay per step (eta_decode_graph_launch); e2e: one graph per "
                           "step of append (reading q, k, v from page-locked host memory) and decode (storing "
                           "out into page-locked host memory) (eta_step_graph_create)"
                           if args.launch == "graph" else "stream launches (eta_decode; e2e: separate calls)"),
                "parallelism": f"replicas x{world} (each rank decodes its own batch)",
            },
            "kernels_ms": {"screen": round(statistics.mean(screen_ms), 6), "attend": round(att_ms, 6),
                           "merge": round(statistics.mean(merge_ms), 6),
                           "note": "second K-step run with library events between the kernels"},
            "roofline": {"kernel": "attend", "bound": "hbm", "achieved": round(achieved, 2),
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": kv_union},
            "step_frac_of_peak": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4),
            "e2e": {"value": round(whole_job_gbs(world, nbytes, e2e), 2), "unit": UNIT,
                    "ms_per_step": round(e2e, 6), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "io": ("the append kernel loads the token's q, k, v rows from pinned host memory and the "
                           "decode stores out into pinned host memory, one graph per token"
                           if args.launch == "graph" else
                           "q, k, v copied from pinned host memory and out copied back by the copy engine")},
            "gpu_launches": 3 * args.steps,
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


def cpu_baseline(wl, args, steps=1, warmup=0):
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits

    s = _oracle_sample(wl)
    summary = oracle.summarize(s.k, s.seq_lens, s.block_size)
    cores = os.cpu_count() or 1
    with threadpool_limits(limits=cores):
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
        for _ in range(warmup):
            _oracle_step(oracle, s, summary)
        ts = []
        for _ in range(steps):
            t0 = time.perf_counter()
            r = _oracle_step(oracle, s, summary)
            ts.append(time.perf_counter() - t0)
    sec = statistics.mean(ts)
    nbytes = _sample_bytes(s, r)
    return {"value": round(nbytes / sec / 1e9, 4), "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "seconds_per_sample": round(sec, 3),
            "sample": (f"{wl.name} seed {wl.seed}: sequence 0, KV head 0 with its {s.n_q_heads} query heads "
                       f"(1/{wl.batch * wl.n_kv_heads} of the step), block metadata precomputed; numpy fp64"),
            "ms_per_step": round(sec * 1e3, 3)}


def run_reference(args):
    rank, _, world = _rank_env()
    if rank != 0:
        return None
    wl = workloads.make(args.workload, args.seed)
    cb = cpu_baseline(wl, args, steps=args.steps, warmup=args.warmup)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": cb["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": cb["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "seed": args.seed,
                   "sample": cb["sample"]},
        "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_prefill(args):
    """Causal forward pass (eta_prefill) over a whole sequence: tensor flops of
    the two contractions over the causal triangle per second, against the
    measured dense bf16 peak.  Not the decode metric; printed on its own line."""
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
    for _ in range(args.steps):
        torch.sum(flush_buf, dim=0, out=flush_sink)
        e0.record(stream)
        eta.eta_prefill(params, stream)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    clk = clocks.stop()
    assert eta.eta_read_device_status(ws) == eta.ETA_OK
    flops = 4.0 * d * (T * (T + 1) / 2) * B * Hq
    t = statistics.mean(ms)
    tflops = flops / (t * 1e-3) / 1e12
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
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t, 4),
        "higher_is_better": True,
        "dtype": "bf16",
        "accum": "f32",
        "data": "synthetic",
        "config": {"workload": f"prefill: batch {B}, {Hq} query / {Hkv} KV heads, seq {T}, d {d}, bf16, learned tau",
                   "flops_per_step": flops,
                   "l2": "flushed before every step by reading a 256 MiB buffer (outside the events)"},
        "roofline": {"kernel": "prefill_tc", "bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                     "peak_kind": kind + " dense bf16 (burst)", "unit": "TFLOP/s", "frac": round(tflops / peak, 4)},
        "gpu_launches": args.steps,
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
    ap.add_argument("--attend-impl", type=int, default=0, choices=[0, 1, 2])
    ap.add_argument("--dense", action="store_true", help="screen off: every block loaded")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="decode step as one recorded CUDA graph (default) or as stream launches")
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
