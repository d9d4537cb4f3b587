"""Python binding of the ETA decode library (libeta.so, sm_100a).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind the C ABI declared in ``include/eta.h``.  PyTorch provides the
device memory and the stream.  The functions mirror the C entry points:

    eta_block_summary_update(...)   refresh per-block metadata after an append
    eta_append_kv(...)              write a new token's K/V and refresh its block
    eta_decode_workspace_size(...)  bytes of scratch for a decode call
    eta_decode(...)                 one decode step (screen, attend, merge)
    eta_read_device_status(...)     read and clear the device status word
    eta_prefill(...) / prefill(...) causal forward pass over whole sequences
    calibration_histogram(...), calibrate_constants(...)
                                    offline per-head threshold calibration
    eta_status_string(code), eta_build_info()

There is no fallback: if libeta.so is missing or fails to load, importing
this package raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeta.so")

ETA_OK = 0
ETA_ERR_INVALID_ARG = 1
ETA_ERR_UNSUPPORTED = 2
ETA_ERR_WORKSPACE = 3
ETA_ERR_CUDA = 4
ETA_ERR_DEVICE_TIMEOUT = 5
ETA_ERR_DEVICE_RANGE = 6
ETA_ERR_DEVICE_LIST = 7

ETA_F32 = 0
ETA_BF16 = 1
ETA_TAU_LEARNED = 0
ETA_TAU_CALIBRATED = 1
ETA_ATTEND_AUTO = 0
ETA_ATTEND_SIMT = 1
ETA_ATTEND_TC = 2
ETA_ATTEND_FUSED = 3


class EtaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {eta_status_string(code)} (status {code})")
        self.code = code


class eta_cache_desc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("block_size", ctypes.c_int), ("max_ctx", ctypes.c_int),
        ("kv_dtype", ctypes.c_int), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("block_table", ctypes.c_void_p), ("num_pages", ctypes.c_int),
    ]


ETA_META_FP16 = 0
ETA_META_FP8 = 1
ETA_META_BOX = 2


class eta_summary_desc(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_void_p), ("sigma", ctypes.c_void_p), ("max_norm", ctypes.c_void_p),
                ("format", ctypes.c_int), ("mu_scale", ctypes.c_void_p), ("sigma_scale", ctypes.c_void_p)]


class eta_decode_params(ctypes.Structure):
    _fields_ = [
        ("cache", eta_cache_desc), ("summary", eta_summary_desc), ("q", ctypes.c_void_p),
        ("tau_mode", ctypes.c_int), ("w_tau", ctypes.c_void_p), ("b_tau", ctypes.c_void_p),
        ("c_tau", ctypes.c_void_p), ("scale", ctypes.c_float), ("beta", ctypes.c_float),
        ("offset_a", ctypes.c_float), ("z", ctypes.c_float), ("n_local_blocks", ctypes.c_int),
        ("screen_enabled", ctypes.c_int), ("attend_impl", ctypes.c_int), ("out", ctypes.c_void_p),
        ("lse", ctypes.c_void_p), ("admitted_count", ctypes.c_void_p), ("union_count", ctypes.c_void_p),
        ("union_list", ctypes.c_void_p), ("union_mask", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("timing_events", ctypes.c_void_p * 4),
        ("trace", ctypes.c_void_p),
    ]


class eta_prefill_params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("seq_len", ctypes.c_int), ("kv_stride", ctypes.c_int),
        ("dtype", ctypes.c_int), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("tau_mode", ctypes.c_int), ("w_tau", ctypes.c_void_p), ("b_tau", ctypes.c_void_p),
        ("c_tau", ctypes.c_void_p), ("scale", ctypes.c_float), ("beta", ctypes.c_float),
        ("offset_a", ctypes.c_float), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("gate_sum", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


PREFILL_WORKSPACE_BYTES = 256  # ETA_PREFILL_WORKSPACE_BYTES in include/eta.h


class eta_calib_params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("seq_len", ctypes.c_int), ("kv_stride", ctypes.c_int),
        ("dtype", ctypes.c_int), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("scale", ctypes.c_float),
        ("lo", ctypes.c_float), ("hi", ctypes.c_float), ("nbins", ctypes.c_int), ("hist", ctypes.c_void_p),
    ]


class eta_step_desc(ctypes.Structure):
    _fields_ = [
        ("decode", ctypes.POINTER(eta_decode_params)), ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p),
        ("positions", ctypes.c_void_p), ("q_new", ctypes.c_void_p), ("h2d_src", ctypes.c_void_p), ("h2d_dst", ctypes.c_void_p),
        ("h2d_bytes", ctypes.c_size_t), ("d2h_src", ctypes.c_void_p), ("d2h_dst", ctypes.c_void_p),
        ("d2h_bytes", ctypes.c_size_t),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run learned_threshold_sparse_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    lib.eta_block_summary_update.argtypes = [P(eta_cache_desc), P(eta_summary_desc), ctypes.c_void_p,
                                             ctypes.c_int, ctypes.c_void_p]
    lib.eta_block_summary_update.restype = ctypes.c_int
    lib.eta_append_kv.argtypes = [P(eta_cache_desc), P(eta_summary_desc), ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p]
    lib.eta_append_kv.restype = ctypes.c_int
    lib.eta_decode_workspace_size.argtypes = [P(eta_decode_params), P(ctypes.c_size_t)]
    lib.eta_decode_workspace_size.restype = ctypes.c_int
    lib.eta_decode.argtypes = [P(eta_decode_params), ctypes.c_void_p]
    lib.eta_decode.restype = ctypes.c_int
    lib.eta_decode_noalloc.argtypes = [P(eta_decode_params), ctypes.c_void_p, ctypes.c_void_p]
    lib.eta_decode_noalloc.restype = ctypes.c_int
    lib.eta_decode_graph_create.argtypes = [P(eta_decode_params), P(ctypes.c_void_p)]
    lib.eta_decode_graph_create.restype = ctypes.c_int
    lib.eta_step_graph_create.argtypes = [P(eta_step_desc), P(ctypes.c_void_p)]
    lib.eta_step_graph_create.restype = ctypes.c_int
    lib.eta_decode_graph_launch.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.eta_decode_graph_launch.restype = ctypes.c_int
    lib.eta_decode_graph_destroy.argtypes = [ctypes.c_void_p]
    lib.eta_decode_graph_destroy.restype = ctypes.c_int
    lib.eta_diag_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.eta_diag_wait_timeout.restype = ctypes.c_int
    lib.eta_read_device_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.eta_read_device_status.restype = ctypes.c_int
    lib.eta_prefill.argtypes = [P(eta_prefill_params), ctypes.c_void_p]
    lib.eta_prefill.restype = ctypes.c_int
    lib.eta_calibration_histogram.argtypes = [P(eta_calib_params), ctypes.c_void_p]
    lib.eta_calibration_histogram.restype = ctypes.c_int
    lib.eta_calibrate_constants.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                            ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    lib.eta_calibrate_constants.restype = ctypes.c_int
    lib.eta_status_string.argtypes = [ctypes.c_int]
    lib.eta_status_string.restype = ctypes.c_char_p
    lib.eta_build_info.argtypes = []
    lib.eta_build_info.restype = ctypes.c_char_p
    return lib


_lib = _load()

SYMBOLS = ("eta_block_summary_update", "eta_append_kv", "eta_decode_workspace_size", "eta_decode", "eta_decode_noalloc",
           "eta_decode_graph_create", "eta_step_graph_create", "eta_decode_graph_launch", "eta_decode_graph_destroy",
           "eta_read_device_status", "eta_diag_wait_timeout", "eta_prefill", "eta_calibration_histogram", "eta_calibrate_constants",
           "eta_status_string", "eta_build_info")

WORKSPACE_CONTROL_BYTES = 69632  # ETA_WORKSPACE_CONTROL_BYTES in include/eta.h
DEVICE_STATUS_TIMEOUT = 1
DEVICE_STATUS_RANGE = 2
DEVICE_STATUS_LIST = 4

ETA_TRACE_SLOTS = 24
TRACE_SLOTS = (("screen_first", 0, True), ("screen_last", 1, False), ("attend_first", 2, True),
               ("attend_last", 3, False), ("tile_first", 4, True), ("merge_first", 6, True),
               ("merge_last", 7, False), ("fused_first", 8, True), ("fused_last", 9, False),
               ("export_first", 10, True), ("export_last", 11, False), ("append_first", 12, True),
               ("append_last", 13, False), ("in_first", 14, True), ("in_last", 15, False),
               ("out_first", 16, True), ("out_last", 17, False))
NOALLOC_SCRATCH_BYTES = 8 << 20  # ETA_NOALLOC_SCRATCH_BYTES in include/eta.h


def library():
    return _lib


def eta_status_string(code: int) -> str:
    return _lib.eta_status_string(int(code)).decode()


def eta_build_info() -> str:
    return _lib.eta_build_info().decode()


# ------------------------------------------------------------ marshalling

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _kv_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return ETA_F32
    if t.dtype == torch.bfloat16:
        return ETA_BF16
    raise TypeError(f"unsupported K/V dtype {t.dtype}")


def cache_desc(k: torch.Tensor, v: torch.Tensor, seq_lens: torch.Tensor, n_q_heads: int,
               block_size: int, block_table: Optional[torch.Tensor] = None) -> eta_cache_desc:
    """Contiguous cache: k, v [B, Hkv, max_ctx, d].  Paged cache: k, v are page
    pools [num_pages, Hkv, block_size, d] and block_table [B, nb_max] int32
    gives each logical block's page (max_ctx = nb_max * block_size)."""
    if block_table is None:
        B, Hkv, Tmax, d = k.shape
        return eta_cache_desc(B, n_q_heads, Hkv, d, block_size, Tmax, _kv_dtype(k), k.data_ptr(), v.data_ptr(),
                              seq_lens.data_ptr())
    P, Hkv, b, d = k.shape
    if b != block_size:
        raise ValueError("page rows must equal block_size")
    B, nbmax = block_table.shape
    c = eta_cache_desc(B, n_q_heads, Hkv, d, block_size, nbmax * block_size, _kv_dtype(k), k.data_ptr(),
                       v.data_ptr(), seq_lens.data_ptr())
    c.block_table = block_table.data_ptr()
    c.num_pages = P
    return c


def alloc_summary(batch: int, n_kv_heads: int, max_ctx: int, head_dim: int, block_size: int,
                  device="cuda", fmt: str = "fp16") -> Dict[str, torch.Tensor]:
    """Metadata buffers: fp16 mu / sigma, or (fmt="fp8") e4m3 codes as uint8
    plus per-block fp32 mu_scale / sigma_scale, or (fmt="box") fp16
    per-coordinate minima / maxima for the comparison box screen (a 0-d "box"
    marker tensor tells the descriptor); fp32 max_norm either way."""
    nb = (max_ctx + block_size - 1) // block_size
    if fmt == "box":
        return {
            "mu": torch.zeros((batch, n_kv_heads, nb, head_dim), dtype=torch.float16, device=device),
            "sigma": torch.zeros((batch, n_kv_heads, nb, head_dim), dtype=torch.float16, device=device),
            "max_norm": torch.zeros((batch, n_kv_heads, nb), dtype=torch.float32, device=device),
            "box": torch.zeros((), dtype=torch.uint8, device=device),
        }
    if fmt == "fp8":
        return {
            "mu": torch.zeros((batch, n_kv_heads, nb, head_dim), dtype=torch.uint8, device=device),
            "sigma": torch.zeros((batch, n_kv_heads, nb, head_dim), dtype=torch.uint8, device=device),
            "max_norm": torch.zeros((batch, n_kv_heads, nb), dtype=torch.float32, device=device),
            "mu_scale": torch.zeros((batch, n_kv_heads, nb), dtype=torch.float32, device=device),
            "sigma_scale": torch.zeros((batch, n_kv_heads, nb), dtype=torch.float32, device=device),
        }
    if fmt != "fp16":
        raise ValueError(fmt)
    return {
        "mu": torch.zeros((batch, n_kv_heads, nb, head_dim), dtype=torch.float16, device=device),
        "sigma": torch.zeros((batch, n_kv_heads, nb, head_dim), dtype=torch.float16, device=device),
        "max_norm": torch.zeros((batch, n_kv_heads, nb), dtype=torch.float32, device=device),
    }


def summary_desc(summary: Dict[str, torch.Tensor]) -> eta_summary_desc:
    d = eta_summary_desc(summary["mu"].data_ptr(), summary["sigma"].data_ptr(), summary["max_norm"].data_ptr())
    if "mu_scale" in summary:
        d.format = ETA_META_FP8
        d.mu_scale = summary["mu_scale"].data_ptr()
        d.sigma_scale = summary["sigma_scale"].data_ptr()
    elif "box" in summary:
        d.format = ETA_META_BOX
    return d


def eta_block_summary_update(k: torch.Tensor, v: torch.Tensor, seq_lens: torch.Tensor,
                             summary: Dict[str, torch.Tensor], block_size: int,
                             first_token: torch.Tensor, max_blocks: int, n_q_heads: Optional[int] = None,
                             stream: Optional[torch.cuda.Stream] = None,
                             block_table: Optional[torch.Tensor] = None) -> None:
    """Recompute the metadata of the blocks at or after first_token[i] (at most
    max_blocks per sequence)."""
    cache = cache_desc(k, v, seq_lens, n_q_heads or k.shape[1], block_size, block_table)
    summ = summary_desc(summary)
    rc = _lib.eta_block_summary_update(ctypes.byref(cache), ctypes.byref(summ),
                                       ctypes.c_void_p(first_token.data_ptr()), int(max_blocks),
                                       _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_block_summary_update")


def eta_append_kv(k: torch.Tensor, v: torch.Tensor, seq_lens: torch.Tensor, summary: Dict[str, torch.Tensor],
                  block_size: int, k_new: torch.Tensor, v_new: torch.Tensor, pos: torch.Tensor,
                  n_q_heads: Optional[int] = None, stream: Optional[torch.cuda.Stream] = None,
                  block_table: Optional[torch.Tensor] = None) -> None:
    """Write k_new / v_new [B, Hkv, d] at row pos[i] of each sequence and refresh
    the summary of the block holding it (seq_lens must already count it)."""
    cache = cache_desc(k, v, seq_lens, n_q_heads or k.shape[1], block_size, block_table)
    summ = summary_desc(summary)
    rc = _lib.eta_append_kv(ctypes.byref(cache), ctypes.byref(summ), ctypes.c_void_p(k_new.data_ptr()),
                            ctypes.c_void_p(v_new.data_ptr()), ctypes.c_void_p(pos.data_ptr()), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_append_kv")


def make_params(q, k, v, seq_lens, summary, block_size, tau_mode, w_tau=None, b_tau=None,
                c_tau=None, scale=None, beta=5.0, offset_a=0.0, z=2.0, n_local_blocks=2,
                screen_enabled=True, attend_impl=ETA_ATTEND_AUTO, out=None, lse=None,
                admitted_count=None, union_count=None, union_list=None, union_mask=None,
                workspace=None, events=None, block_table=None, trace=None) -> eta_decode_params:
    B, Hq, d = q.shape
    p = eta_decode_params()
    p.cache = cache_desc(k, v, seq_lens, Hq, block_size, block_table)
    if summary is not None:
        p.summary = summary_desc(summary)
    p.q = q.data_ptr()
    p.tau_mode = ETA_TAU_LEARNED if tau_mode in ("learned", ETA_TAU_LEARNED) else ETA_TAU_CALIBRATED
    p.w_tau = None if w_tau is None else w_tau.data_ptr()
    p.b_tau = None if b_tau is None else b_tau.data_ptr()
    p.c_tau = None if c_tau is None else c_tau.data_ptr()
    p.scale = float(1.0 / math.sqrt(d) if scale is None else scale)
    p.beta = float(beta)
    p.offset_a = float(offset_a)
    p.z = float(z)
    p.n_local_blocks = int(n_local_blocks)
    p.screen_enabled = 1 if screen_enabled else 0
    p.attend_impl = int(attend_impl)
    p.out = None if out is None else out.data_ptr()
    p.lse = None if lse is None else lse.data_ptr()
    p.admitted_count = None if admitted_count is None else admitted_count.data_ptr()
    p.union_count = None if union_count is None else union_count.data_ptr()
    p.union_list = None if union_list is None else union_list.data_ptr()
    p.union_mask = None if union_mask is None else union_mask.data_ptr()
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    if events is not None:
        for j, e in enumerate(events):
            if e is not None and not e.cuda_event:
                e.record()  # torch creates the underlying cudaEvent_t lazily
            p.timing_events[j] = None if e is None else e.cuda_event
    if trace is not None:
        if trace.dtype != torch.int64 or trace.numel() < ETA_TRACE_SLOTS or not trace.is_cuda:
            raise ValueError("trace: a CUDA int64 tensor of at least ETA_TRACE_SLOTS elements")
        p.trace = trace.data_ptr()
    return p


def trace_times(trace: torch.Tensor) -> dict:
    """Decode a step trace (see include/eta.h) into nanosecond times by name;
    slots no kernel wrote are left out."""
    raw = [int(x) & 0xFFFFFFFFFFFFFFFF for x in trace[:ETA_TRACE_SLOTS].cpu().tolist()]
    out = {}
    for name, slot, first in TRACE_SLOTS:
        v = raw[slot]
        if v:
            out[name] = (~v & 0xFFFFFFFFFFFFFFFF) if first else v
    return out


def eta_decode_workspace_size(params: eta_decode_params) -> int:
    n = ctypes.c_size_t(0)
    rc = _lib.eta_decode_workspace_size(ctypes.byref(params), ctypes.byref(n))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_decode_workspace_size")
    return int(n.value)


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace (the leading status word must start at zero)."""
    return torch.zeros(((nbytes + 255) // 256) * 256, dtype=torch.uint8, device=device)


def eta_decode(params: eta_decode_params, stream: Optional[torch.cuda.Stream] = None) -> None:
    rc = _lib.eta_decode(ctypes.byref(params), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_decode")


def eta_decode_noalloc(params: eta_decode_params, device_status: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None) -> None:
    """eta_decode without a caller workspace, for callers that cannot allocate
    device memory: the library's fixed device scratch is used instead (see
    include/eta.h).  Calls sharing that scratch must not overlap on the GPU.
    device_status (an int32 device tensor, optional) receives the step's
    device status bits (DEVICE_STATUS_TIMEOUT, DEVICE_STATUS_RANGE, DEVICE_STATUS_LIST)."""
    ptr = None if device_status is None else device_status.data_ptr()
    rc = _lib.eta_decode_noalloc(ctypes.byref(params), ptr, _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_decode_noalloc")


def eta_decode_graph_create(params: eta_decode_params) -> int:
    """Record one decode step with these parameters into a CUDA graph; returns
    the graph handle (see include/eta.h: the buffers params points to must
    stay in place while the graph lives, their contents may change)."""
    h = ctypes.c_void_p()
    rc = _lib.eta_decode_graph_create(ctypes.byref(params), ctypes.byref(h))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_decode_graph_create")
    return int(h.value)


def eta_step_graph_create(desc: eta_step_desc) -> int:
    """Record one serving-loop token (input copy, KV append, decode, output
    copy; see include/eta.h) into a CUDA graph; returns the graph handle."""
    h = ctypes.c_void_p()
    rc = _lib.eta_step_graph_create(ctypes.byref(desc), ctypes.byref(h))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_step_graph_create")
    return int(h.value)


def eta_decode_graph_launch(handle: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    rc = _lib.eta_decode_graph_launch(ctypes.c_void_p(handle), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_decode_graph_launch")


def eta_decode_graph_destroy(handle: int) -> None:
    rc = _lib.eta_decode_graph_destroy(ctypes.c_void_p(handle))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_decode_graph_destroy")


class DecodeGraph:
    """Owner of a recorded decode step: keeps the parameter block and the
    tensors it points to alive, launches the graph, releases it on close()."""

    def __init__(self, params: eta_decode_params, tensors=()):
        self.params = params
        self._keep = list(tensors)
        self.handle = 0
        self.handle = eta_decode_graph_create(params)

    def launch(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        if not self.handle:
            raise EtaError(ETA_ERR_INVALID_ARG, "eta_decode_graph_launch")
        eta_decode_graph_launch(self.handle, stream)

    def close(self) -> None:
        if self.handle:
            h, self.handle = self.handle, 0
            eta_decode_graph_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class StepGraph(DecodeGraph):
    """Owner of a recorded serving-loop token: the host-to-device copy of
    `h2d` (page-locked host tensor) into `h2d_dst`, the append of k_new / v_new
    at `positions` with the queries q_new copied into the decode's q
    (optional; the new rows may be page-locked host tensors), the decode step
    of `params`, and the copy of `d2h_src` into the page-locked host tensor
    `d2h`."""

    def __init__(self, params: eta_decode_params, *, k_new=None, v_new=None, positions=None, q_new=None, h2d=None,
                 h2d_dst=None, d2h_src=None, d2h=None, tensors=()):
        self.params = params
        self._keep = [t for t in (k_new, v_new, positions, q_new, h2d, h2d_dst, d2h_src, d2h) if t is not None]
        self._keep += list(tensors)
        d = eta_step_desc()
        d.decode = ctypes.pointer(params)
        d.k_new, d.v_new, d.positions, d.q_new = _ptr(k_new), _ptr(v_new), _ptr(positions), _ptr(q_new)
        if h2d is not None:
            d.h2d_src, d.h2d_dst = _ptr(h2d), _ptr(h2d_dst)
            d.h2d_bytes = h2d.numel() * h2d.element_size()
        if d2h is not None:
            d.d2h_src, d.d2h_dst = _ptr(d2h_src), _ptr(d2h)
            d.d2h_bytes = d2h.numel() * d2h.element_size()
        self.desc = d
        self.handle = 0
        self.handle = eta_step_graph_create(d)


def eta_diag_wait_timeout(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Diagnostic: a bounded device-side wait that nothing completes gives up
    and sets the workspace's timeout bit (see include/eta.h)."""
    rc = _lib.eta_diag_wait_timeout(ctypes.c_void_p(workspace.data_ptr()), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_diag_wait_timeout")


def eta_read_device_status(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    return int(_lib.eta_read_device_status(ctypes.c_void_p(workspace.data_ptr()), _stream_handle(stream)))


def decode(q, k, v, seq_lens, summary, block_size, tau_mode, *, w_tau=None, b_tau=None, c_tau=None,
           scale=None, beta=5.0, offset_a=0.0, z=2.0, n_local_blocks=2, screen_enabled=True,
           attend_impl=ETA_ATTEND_AUTO, selection=False, workspace=None, out=None, lse=None,
           events=None, stream=None, block_table=None, trace=None) -> Dict[str, torch.Tensor]:
    """Allocate outputs (and the workspace if not given) with torch and run one
    decode step.  Returns {"out", "lse", "workspace"} plus, with selection=True,
    {"admitted_count", "union_count", "union_list", "union_mask"}.  `trace`:
    an optional zeroed int64 device tensor of ETA_TRACE_SLOTS elements that
    receives the step trace (read it with trace_times)."""
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    nb = block_table.shape[1] if block_table is not None else (k.shape[2] + block_size - 1) // block_size
    dev = q.device
    res = {"out": out if out is not None else torch.empty_like(q),
           "lse": lse if lse is not None else torch.empty((B, Hq), dtype=torch.float32, device=dev)}
    if selection:
        res["admitted_count"] = torch.empty((B, Hq), dtype=torch.int32, device=dev)
        res["union_count"] = torch.empty((B, Hkv), dtype=torch.int32, device=dev)
        res["union_list"] = torch.empty((B, Hkv, nb), dtype=torch.int32, device=dev)
        res["union_mask"] = torch.empty((B, Hkv, nb), dtype=torch.int32, device=dev)
    kw = dict(w_tau=w_tau, b_tau=b_tau, c_tau=c_tau, scale=scale, beta=beta, offset_a=offset_a, z=z,
              n_local_blocks=n_local_blocks, screen_enabled=screen_enabled, attend_impl=attend_impl,
              out=res["out"], lse=res["lse"], admitted_count=res.get("admitted_count"),
              union_count=res.get("union_count"), union_list=res.get("union_list"),
              union_mask=res.get("union_mask"), events=events, block_table=block_table, trace=trace)
    params = make_params(q, k, v, seq_lens, summary, block_size, tau_mode, **kw)
    if workspace is None:
        workspace = alloc_workspace(eta_decode_workspace_size(params), dev)
    params.workspace = workspace.data_ptr()
    params.workspace_bytes = workspace.numel()
    eta_decode(params, stream)
    res["workspace"] = workspace
    return res


# ------------------------------------------------------------ causal forward

def make_prefill_params(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_len: int, tau_mode: str, *,
                        w_tau=None, b_tau=None, c_tau=None, scale: Optional[float] = None, beta: float = 5.0,
                        offset_a: float = 0.0, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                        gate_sum: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None) -> eta_prefill_params:
    """q [B, Hq, T, d], k and v [B, Hkv, kv_stride, d] (kv_stride >= T), all
    bf16 on the device; out like q."""
    B, Hq, T, d = q.shape
    p = eta_prefill_params()
    p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim = B, Hq, k.shape[1], d
    p.seq_len, p.kv_stride = int(seq_len), k.shape[2]
    p.dtype = _kv_dtype(q)
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.tau_mode = ETA_TAU_LEARNED if tau_mode == "learned" else ETA_TAU_CALIBRATED
    p.w_tau = None if w_tau is None else w_tau.data_ptr()
    p.b_tau = None if b_tau is None else b_tau.data_ptr()
    p.c_tau = None if c_tau is None else c_tau.data_ptr()
    p.scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    p.beta = float(beta)
    p.offset_a = float(offset_a)
    p.out = out.data_ptr()
    p.lse = None if lse is None else lse.data_ptr()
    p.gate_sum = None if gate_sum is None else gate_sum.data_ptr()
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel()
    return p


def eta_prefill(params: eta_prefill_params, stream: Optional[torch.cuda.Stream] = None) -> None:
    rc = _lib.eta_prefill(ctypes.byref(params), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_prefill")


def prefill(q, k, v, seq_len: int, tau_mode: str, *, w_tau=None, b_tau=None, c_tau=None, scale=None, beta=5.0,
            offset_a=0.0, stream=None) -> Dict[str, torch.Tensor]:
    """Allocate the outputs and a workspace, run eta_prefill; returns out, lse,
    gate_sum and the workspace (for eta_read_device_status)."""
    out = torch.empty_like(q)
    B, Hq, T, _ = q.shape
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    gate = torch.empty_like(lse)
    ws = alloc_workspace(PREFILL_WORKSPACE_BYTES, q.device)
    p = make_prefill_params(q, k, v, seq_len, tau_mode, w_tau=w_tau, b_tau=b_tau, c_tau=c_tau, scale=scale,
                            beta=beta, offset_a=offset_a, out=out, lse=lse, gate_sum=gate, workspace=ws)
    eta_prefill(p, stream)
    return {"out": out, "lse": lse, "gate_sum": gate, "workspace": ws}


# ------------------------------------------------------------ calibration

def calibration_histogram(q: torch.Tensor, k: torch.Tensor, seq_len: int, *, scale: Optional[float] = None,
                          lo: float = -8.0, hi: float = 8.0, nbins: int = 4096,
                          hist: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Add the 1/(t+1)-weighted causal logit histogram of every query head of
    q [B, Hq, T, d] against k [B, Hkv, kv_stride, d] to ``hist`` (fp64
    [Hq, nbins + 2], allocated zeroed when not given) and return it."""
    B, Hq, T, d = q.shape
    if hist is None:
        hist = torch.zeros((Hq, nbins + 2), dtype=torch.float64, device=q.device)
    p = eta_calib_params()
    p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim = B, Hq, k.shape[1], d
    p.seq_len, p.kv_stride = int(seq_len), k.shape[2]
    p.dtype = _kv_dtype(q)
    p.q, p.k = q.data_ptr(), k.data_ptr()
    p.scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    p.lo, p.hi, p.nbins = float(lo), float(hi), int(nbins)
    p.hist = hist.data_ptr()
    rc = _lib.eta_calibration_histogram(ctypes.byref(p), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_calibration_histogram")
    return hist


def calibrate_constants(hist: torch.Tensor, lo: float, hi: float, target) -> "np.ndarray":
    """Per-head effective thresholds tau~ reaching the target densities (host
    solver over a histogram from calibration_histogram)."""
    import numpy as np

    h = np.ascontiguousarray(hist.detach().cpu().numpy(), dtype=np.float64)
    n, nb2 = h.shape
    tgt = np.ascontiguousarray(np.broadcast_to(np.asarray(target, dtype=np.float32), (n,)))
    c = np.zeros(n, np.float32)
    rc = _lib.eta_calibrate_constants(h.ctypes.data, n, nb2 - 2, float(lo), float(hi), tgt.ctypes.data,
                                      c.ctypes.data)
    if rc != ETA_OK:
        raise EtaError(rc, "eta_calibrate_constants")
    return c


def eta_calibration_histogram(params: eta_calib_params, stream: Optional[torch.cuda.Stream] = None) -> None:
    rc = _lib.eta_calibration_histogram(ctypes.byref(params), _stream_handle(stream))
    if rc != ETA_OK:
        raise EtaError(rc, "eta_calibration_histogram")


def eta_calibrate_constants(hist_host, n_heads: int, nbins: int, lo: float, hi: float, target_host, c_host) -> None:
    """Host arrays (numpy): hist [n_heads, nbins + 2] float64, target and c
    [n_heads] float32 (c written)."""
    rc = _lib.eta_calibrate_constants(hist_host.ctypes.data, int(n_heads), int(nbins), float(lo), float(hi),
                                      target_host.ctypes.data, c_host.ctypes.data)
    if rc != ETA_OK:
        raise EtaError(rc, "eta_calibrate_constants")
