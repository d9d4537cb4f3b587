"""Seeded synthetic inputs for the ETA decode step.

This module is shared by the CPU oracle side (tests, threshold calibration
script) and the CUDA side (tests, bench).  It holds only random draws and the
planted structure of each workload; none of the method's arithmetic (block
summaries, block bounds, tempering, softmax) lives here.

Workload shapes follow the decode benchmarks of "Elastic Threshold Attention:
Learned Contextual Sparsity for Long-Context Decoding" (section 4.8, Table 5
caption; Appendix F.3, Table 10 caption): single-token queries, GQA with
H_Q / H_KV query heads per KV head, head_dim 64 or 128, KV blocks of 64 or 128
tokens, contexts up to 512K.

Per-head thresholds that make a workload hit a target admitted density are
input data: they are stored in ``tests/golden/thresholds.json`` and written by
``tests/golden/make_thresholds.py``, which calls only the CPU oracle.
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import json
import math
import os
from typing import List, Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
THRESHOLDS_JSON = os.path.join(os.path.dirname(_HERE), "tests", "golden", "thresholds.json")

F32 = "f32"
BF16 = "bf16"
TAU_LEARNED = "learned"
TAU_CALIBRATED = "calibrated"


@dataclasses.dataclass
class Workload:
    """One decode step's inputs.

    Tensors live on the host.  ``k``/``v`` are ``[B, Hkv, max_ctx, d]`` and ``q``
    is ``[B, Hq, d]`` in the KV dtype (``torch.float32`` or ``torch.bfloat16``);
    rows of ``k``/``v`` at positions ``>= seq_lens[i]`` are zero.  Threshold
    parameters are fp32: ``w_tau [Hq, d]``, ``b_tau [Hq]`` in learned mode,
    ``c_tau [Hq]`` in calibrated mode.
    """

    name: str
    seed: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int
    max_ctx: int
    seq_lens: List[int]
    dtype: str
    tau_mode: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    w_tau: Optional[np.ndarray]
    b_tau: Optional[np.ndarray]
    c_tau: Optional[np.ndarray]
    scale: float
    beta: float = 5.0
    offset_a: float = 0.0
    z: float = 2.0
    n_local_blocks: int = 2
    screen_enabled: bool = True
    # planted structure, for assertions (block ids per (seq, q head))
    planted: Optional[dict] = None
    target_union_density: Optional[float] = None

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    def n_blocks(self, i: int) -> int:
        return (self.seq_lens[i] + self.block_size - 1) // self.block_size

    @property
    def nb_max(self) -> int:
        return (self.max_ctx + self.block_size - 1) // self.block_size

    def with_params(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# ---------------------------------------------------------------- helpers

def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


_CHUNK = 1 << 22


def _normal_big(key, shape, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) float32 array filled in parallel: element block j (of 2^22
    elements, row-major) comes from its own PCG64 stream seeded with key + [j],
    so the values do not depend on the thread count."""
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)

    def fill(j):
        lo, hi = j * _CHUNK, min(n, (j + 1) * _CHUNK)
        out[lo:hi] = np.random.default_rng(list(key) + [j]).standard_normal(size=hi - lo, dtype=np.float32)

    nblk = (n + _CHUNK - 1) // _CHUNK
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, os.cpu_count() or 1))) as ex:
        list(ex.map(fill, range(nblk)))
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def _to_kv(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t if dtype == F32 else t.to(torch.bfloat16)


def _group_queries(rng, batch, hq, hkv, d, rho: float) -> np.ndarray:
    """Queries with unit-variance coordinates; heads that share a KV head share
    a common component with correlation ``rho``."""
    g = hq // hkv
    shared = _normal(rng, (batch, hkv, 1, d))
    own = _normal(rng, (batch, hkv, g, d))
    q = math.sqrt(rho) * shared + math.sqrt(1.0 - rho) * own
    return q.reshape(batch, hq, d).astype(np.float32)


def _aligned_keys(rng, keys: np.ndarray, direction: np.ndarray, cos_lo: float, cos_hi: float) -> np.ndarray:
    """Rotate each row of ``keys`` toward ``direction`` so that its cosine with it
    is drawn U[cos_lo, cos_hi], keeping the row's norm."""
    u = direction / np.linalg.norm(direction)
    norms = np.linalg.norm(keys, axis=1, keepdims=True)
    along = keys @ u
    perp = keys - along[:, None] * u[None, :]
    perp /= np.maximum(np.linalg.norm(perp, axis=1, keepdims=True), 1e-12)
    c = rng.uniform(cos_lo, cos_hi, size=(keys.shape[0], 1)).astype(np.float32)
    s = np.sqrt(1.0 - c * c)
    return (norms * (c * u[None, :] + s * perp)).astype(np.float32)


def _load_thresholds(name: str, seed: int) -> Optional[dict]:
    if not os.path.exists(THRESHOLDS_JSON):
        return None
    with open(THRESHOLDS_JSON) as f:
        table = json.load(f)
    return table.get(name, {}).get(f"seed{seed}")


def _screenable_positions(nb: int, n_local_blocks: int) -> int:
    """Number of leading blocks that are not in the always-loaded recent window."""
    return max(0, nb - 1 - max(n_local_blocks, 0))


# ---------------------------------------------------------------- configs

def tiny(seed: int = 0) -> Workload:
    """Batch 1, 4 heads (no GQA), d 64, context 4096, block 64, fp32.  q, K, V ~
    N(0,1); W_tau ~ N(0, 1/64), b_tau = 0.5; 3 planted blocks per head whose keys
    are 2 q + N(0, 0.1^2)."""
    rng = np.random.default_rng([1, seed])
    B, H, d, T, b = 1, 4, 64, 4096, 64
    q = _normal(rng, (B, H, d))
    k = _normal(rng, (B, H, T, d))
    v = _normal(rng, (B, H, T, d))
    nb = T // b
    planted = {}
    for h in range(H):
        blocks = rng.choice(_screenable_positions(nb, 2), size=3, replace=False)
        planted[(0, h)] = sorted(int(x) for x in blocks)
        for blk in blocks:
            rows = slice(blk * b, (blk + 1) * b)
            k[0, h, rows] = 2.0 * q[0, h][None, :] + _normal(rng, (b, d), 0.1)
    w_tau = _normal(rng, (H, d), 1.0 / 8.0)
    b_tau = np.full((H,), 0.5, np.float32)
    return Workload(name="c1_tiny", seed=seed, batch=B, n_q_heads=H, n_kv_heads=H,
                    head_dim=d, block_size=b, max_ctx=T, seq_lens=[T], dtype=F32,
                    tau_mode=TAU_LEARNED, q=_to_kv(q, F32), k=_to_kv(k, F32),
                    v=_to_kv(v, F32), w_tau=w_tau, b_tau=b_tau, c_tau=None,
                    scale=1.0 / math.sqrt(d), planted=planted)


def single(seed: int = 0, T: int = 32768) -> Workload:
    """Batch 1, 16 query / 4 KV heads, d 128, context 32768, block 64, bf16,
    learned tau.  Keys ~ N(0,1) with 5% of the blocks planted: every key of a
    planted block is turned toward one seeded query head of its group with a
    cosine drawn U[0.6, 0.9]."""
    rng = np.random.default_rng([2, seed])
    B, Hq, Hkv, d, b = 1, 16, 4, 128, 64
    G = Hq // Hkv
    q = _group_queries(rng, B, Hq, Hkv, d, 0.5)
    k = _normal_big([2, seed, 0], (B, Hkv, T, d))
    v = _normal_big([2, seed, 1], (B, Hkv, T, d))
    nb = (T + b - 1) // b
    n_plant = max(1, round(0.05 * nb))
    planted = {}
    for g in range(Hkv):
        blocks = rng.choice(_screenable_positions(nb, 2), size=n_plant, replace=False)
        heads = rng.integers(0, G, size=n_plant)
        for blk, hh in zip(blocks, heads):
            h = g * G + int(hh)
            planted.setdefault((0, h), []).append(int(blk))
            rows = slice(blk * b, min((blk + 1) * b, T))
            k[0, g, rows] = _aligned_keys(rng, k[0, g, rows], q[0, h], 0.6, 0.9)
    w_tau = _normal(rng, (Hq, d), 0.1 / math.sqrt(d))
    wl = Workload(name="c2_single", seed=seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv,
                  head_dim=d, block_size=b, max_ctx=T, seq_lens=[T], dtype=BF16,
                  tau_mode=TAU_LEARNED, q=_to_kv(q, BF16), k=_to_kv(k, BF16),
                  v=_to_kv(v, BF16), w_tau=w_tau, b_tau=None, c_tau=None,
                  scale=1.0 / math.sqrt(d), planted={kk: sorted(vv) for kk, vv in planted.items()},
                  target_union_density=0.38)
    return wl


def _cluster_keys(rng, T: int, d: int, b: int, n_centres: int = 64, spread: float = 0.3,
                  noise_key=None) -> np.ndarray:
    centres = _normal(rng, (n_centres, d))
    nb = (T + b - 1) // b
    pick = rng.integers(0, n_centres, size=nb)
    per_token = np.repeat(pick, b)[:T]
    keys = centres[per_token]
    keys += _normal(rng, (T, d), spread) if noise_key is None else _normal_big(noise_key, (T, d), spread)
    return keys


def long(seed: int = 0, T: int = 131072) -> Workload:
    """Batch 1, 16 query / 4 KV heads, d 128, context 131072, block 64, bf16.
    Each block's keys come from one of 64 random cluster centres (N(0, I))
    plus 0.3 N(0, I) noise; V ~ N(0,1).  Per-head constant thresholds
    (calibrated mode)."""
    rng = np.random.default_rng([3, seed])
    B, Hq, Hkv, d, b = 1, 16, 4, 128, 64
    q = _group_queries(rng, B, Hq, Hkv, d, 0.5)
    k = np.stack([_cluster_keys(rng, T, d, b, noise_key=[3, seed, 0, g]) for g in range(Hkv)])[None]
    v = _normal_big([3, seed, 1], (B, Hkv, T, d))
    wl = Workload(name="c3_long", seed=seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv,
                  head_dim=d, block_size=b, max_ctx=T, seq_lens=[T], dtype=BF16,
                  tau_mode=TAU_CALIBRATED, q=_to_kv(q, BF16), k=_to_kv(k, BF16),
                  v=_to_kv(v, BF16), w_tau=None, b_tau=None, c_tau=None,
                  scale=1.0 / math.sqrt(d), target_union_density=0.38)
    return wl


def max_context(seed: int = 0, T: int = 524288) -> Workload:
    """Batch 1, 16 query / 4 KV heads, d 128, context 524288, block 128, bf16,
    learned tau.  K, V ~ N(0,1) plus one needle block per query head at a seeded
    position whose keys are turned toward that head's query (cosine U[0.8, 0.95])."""
    rng = np.random.default_rng([4, seed])
    B, Hq, Hkv, d, b = 1, 16, 4, 128, 128
    G = Hq // Hkv
    q = _group_queries(rng, B, Hq, Hkv, d, 0.5)
    k = _normal_big([4, seed, 0], (B, Hkv, T, d))
    v = _normal_big([4, seed, 1], (B, Hkv, T, d))
    nb = (T + b - 1) // b
    planted = {}
    for g in range(Hkv):
        blocks = rng.choice(_screenable_positions(nb, 2), size=G, replace=False)
        for j, blk in enumerate(blocks):
            h = g * G + j
            planted[(0, h)] = [int(blk)]
            rows = slice(blk * b, (blk + 1) * b)
            k[0, g, rows] = _aligned_keys(rng, k[0, g, rows], q[0, h], 0.8, 0.95)
    w_tau = _normal(rng, (Hq, d), 0.1 / math.sqrt(d))
    wl = Workload(name="c4_max", seed=seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv,
                  head_dim=d, block_size=b, max_ctx=T, seq_lens=[T], dtype=BF16,
                  tau_mode=TAU_LEARNED, q=_to_kv(q, BF16), k=_to_kv(k, BF16),
                  v=_to_kv(v, BF16), w_tau=w_tau, b_tau=None, c_tau=None,
                  scale=1.0 / math.sqrt(d), planted=planted, target_union_density=0.38)
    return wl


def batched(seed: int = 0, batch: int = 8, t_lo: int = 16384, t_hi: int = 131072) -> Workload:
    """Batch 8, 16 query / 4 KV heads, d 128, contexts drawn U[16384, 131072]
    per sequence, block 64, bf16, cluster keys as in the long-context case,
    calibrated mode with per-head constants drawn U[0.5, 2.0]."""
    rng = np.random.default_rng([5, seed])
    B, Hq, Hkv, d, b = batch, 16, 4, 128, 64
    lens = [int(x) for x in rng.integers(t_lo, t_hi + 1, size=B)]
    Tmax = t_hi
    q = _group_queries(rng, B, Hq, Hkv, d, 0.5)
    k = torch.zeros((B, Hkv, Tmax, d), dtype=torch.bfloat16)
    v = torch.zeros((B, Hkv, Tmax, d), dtype=torch.bfloat16)
    for i, T in enumerate(lens):
        for g in range(Hkv):
            k[i, g, :T] = _to_kv(_cluster_keys(rng, T, d, b, noise_key=[5, seed, 0, i, g]), BF16)
            v[i, g, :T] = _to_kv(_normal_big([5, seed, 1, i, g], (T, d)), BF16)
    # drawn here; the stored constants move each draw into a guard-banded gap
    # of that head's block scores (tests/golden/make_thresholds.py)
    c_tau = rng.uniform(0.5, 2.0, size=Hq).astype(np.float32)
    return Workload(name="c5_batched", seed=seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv,
                    head_dim=d, block_size=b, max_ctx=Tmax, seq_lens=lens, dtype=BF16,
                    tau_mode=TAU_CALIBRATED, q=_to_kv(q, BF16), k=k, v=v, w_tau=None,
                    b_tau=None, c_tau=c_tau, scale=1.0 / math.sqrt(d))


def custom(seed: int, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
           block_size: int, seq_lens: List[int], dtype: str = BF16,
           tau_mode: str = TAU_LEARNED, max_ctx: Optional[int] = None,
           key_kind: str = "normal", tau_bias: float = 1.8, tau_std: float = 0.0,
           rho: float = 0.5) -> Workload:
    """Small seeded case for edge-case tests.  ``key_kind`` is ``normal`` or
    ``cluster``.  Learned mode draws W_tau ~ N(0, tau_std^2 / d) and sets b_tau to
    ``tau_bias``; calibrated mode sets c_tau to ``tau_bias`` plus a per-head
    U[-0.2, 0.2] spread."""
    rng = np.random.default_rng([6, seed])
    B, Hq, Hkv, d, b = batch, n_q_heads, n_kv_heads, head_dim, block_size
    Tmax = max_ctx if max_ctx is not None else max(1, max(seq_lens))
    q = _group_queries(rng, B, Hq, Hkv, d, rho)
    k = np.zeros((B, Hkv, Tmax, d), np.float32)
    v = np.zeros((B, Hkv, Tmax, d), np.float32)
    for i, T in enumerate(seq_lens):
        for g in range(Hkv):
            if T == 0:
                continue
            if key_kind == "cluster":
                k[i, g, :T] = _cluster_keys(rng, T, d, b)
            else:
                k[i, g, :T] = _normal(rng, (T, d))
            v[i, g, :T] = _normal(rng, (T, d))
    if tau_mode == TAU_LEARNED:
        w_tau = _normal(rng, (Hq, d), tau_std / math.sqrt(d)) if tau_std > 0 else np.zeros((Hq, d), np.float32)
        b_tau = np.full((Hq,), tau_bias, np.float32)
        c_tau = None
    else:
        w_tau = b_tau = None
        c_tau = (tau_bias + rng.uniform(-0.2, 0.2, size=Hq)).astype(np.float32)
    return Workload(name=f"custom_{seed}", seed=seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv,
                    head_dim=d, block_size=b, max_ctx=Tmax, seq_lens=list(seq_lens), dtype=dtype,
                    tau_mode=tau_mode, q=_to_kv(q, dtype), k=_to_kv(k, dtype), v=_to_kv(v, dtype),
                    w_tau=w_tau, b_tau=b_tau, c_tau=c_tau, scale=1.0 / math.sqrt(d))


@dataclasses.dataclass
class PrefillInputs:
    """Inputs of one causal forward pass over whole sequences: ``q``
    ``[B, Hq, T, d]``, ``k``/``v`` ``[B, Hkv, kv_stride, d]`` (bf16, host) and
    fp32 threshold parameters as in ``Workload``."""

    seed: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_len: int
    kv_stride: int
    tau_mode: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    w_tau: Optional[np.ndarray]
    b_tau: Optional[np.ndarray]
    c_tau: Optional[np.ndarray]
    scale: float
    beta: float = 5.0
    offset_a: float = 0.0


def prefill_case(seed: int, batch: int, n_q_heads: int, n_kv_heads: int, seq_len: int,
                 kv_stride: Optional[int] = None, head_dim: int = 128, tau_mode: str = TAU_LEARNED,
                 tau_bias: float = 0.5, tau_std: float = 1.0, key_ramp: float = 0.0,
                 tail_fill: float = 0.0, beta: float = 5.0, offset_a: float = 0.0) -> PrefillInputs:
    """Seeded prefill inputs.  q, k, v ~ N(0, 1); with ``key_ramp`` > 0 key j
    is scaled by 1 + key_ramp j / T, so the logits grow along the sequence.
    Rows of k and v at positions >= seq_len (up to ``kv_stride``) hold
    ``tail_fill`` (NaN allowed).  Learned mode: W_tau ~ N(0, tau_std^2 / d),
    b_tau = tau_bias; calibrated: c_tau = tau_bias + U[-0.2, 0.2] per head."""
    rng = np.random.default_rng([7, seed])
    B, Hq, Hkv, T, d = batch, n_q_heads, n_kv_heads, seq_len, head_dim
    S = kv_stride if kv_stride is not None else T
    q = rng.standard_normal((B, Hq, T, d), dtype=np.float32)
    k = np.full((B, Hkv, S, d), tail_fill, np.float32)
    v = np.full((B, Hkv, S, d), tail_fill, np.float32)
    k[:, :, :T] = rng.standard_normal((B, Hkv, T, d), dtype=np.float32)
    v[:, :, :T] = rng.standard_normal((B, Hkv, T, d), dtype=np.float32)
    if key_ramp:
        k[:, :, :T] *= (1.0 + key_ramp * np.arange(T, dtype=np.float32) / T)[None, None, :, None]
    if tau_mode == TAU_LEARNED:
        w_tau = _normal(rng, (Hq, d), tau_std / math.sqrt(d))
        b_tau = np.full((Hq,), tau_bias, np.float32)
        c_tau = None
    else:
        w_tau = b_tau = None
        c_tau = (tau_bias + rng.uniform(-0.2, 0.2, size=Hq)).astype(np.float32)
    return PrefillInputs(seed=seed, batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=T, kv_stride=S,
                         tau_mode=tau_mode, q=_to_kv(q, BF16), k=_to_kv(k, BF16), v=_to_kv(v, BF16),
                         w_tau=w_tau, b_tau=b_tau, c_tau=c_tau, scale=1.0 / math.sqrt(d), beta=beta,
                         offset_a=offset_a)


def _attach_thresholds(wl: Workload) -> Workload:
    entry = _load_thresholds(wl.name, wl.seed)
    if entry is None:
        return wl
    if wl.tau_mode == TAU_LEARNED:
        return wl.with_params(b_tau=np.asarray(entry["b_tau"], np.float32))
    return wl.with_params(c_tau=np.asarray(entry["c_tau"], np.float32))


CONFIGS = {
    "c1_tiny": tiny,
    "c2_single": single,
    "c3_long": long,
    "c4_max": max_context,
    "c5_batched": batched,
}


def make(name: str, seed: int = 0, raw_thresholds: bool = False, **kw) -> Workload:
    """Workload `name` with its stored thresholds (tests/golden/thresholds.json)
    applied; raw_thresholds=True keeps the generator's own draws (the input of
    the script that writes that file)."""
    wl = CONFIGS[name](seed=seed, **kw)
    return wl if raw_thresholds else _attach_thresholds(wl)
