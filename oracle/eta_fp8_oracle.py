"""CPU oracle for the FP8 block metadata of the ETA screen: the centroid and
spread stored in 8-bit floats with a per-block scale, which halves the bytes
the screen reads for every block (section 5, Limitations and Conclusion,
names FP8 metadata quantization as a systems extension; the format below,
e4m3 codes with one fp32 scale per block and field, is this project's
reading).

TEST INFRASTRUCTURE ONLY.  Only the test suite may import or run this module.
It shares no code with the CUDA library and does not import it.

What is stored per (block, KV head), following Appendix F.1 of "Elastic
Threshold Attention: Learned Contextual Sparsity for Long-Context Decoding"
with its fp16 fields replaced by scaled e4m3:
  mu_code [d] e4m3, mu_scale fp32    with mu~ = e4m3(mu / mu_scale) mu_scale,
  sigma_code [d] e4m3, sigma_scale   likewise for the coordinate spread,
  M fp32                             max ||k - mu~|| over the block's keys,
                                     measured from the dequantised centroid
                                     and rounded up, so the geometric half of
                                     the bound stays a true upper bound.
The scale maps the largest magnitude of the block to 448, the largest finite
e4m3 value.

Where floating point decides a code, this oracle takes the decision in the
kernel's precision: the centroid and spread are accumulated in fp32, one
correctly rounded operation at a time in the kernel's order (rows in order;
two passes), the scale and the quotients are fp32 divisions, and the code is
the nearest e4m3 value (ties to even, saturating at 448).  M is computed in
float64 and rounded up to fp32.

Parity status: pinned by tests/test_oracle_fp8_pins.py (the e4m3 rounding
against a brute-force nearest-value search over all 256 codes, closed forms of
the scale and of a constant block, the strict bound by brute force, agreement
of the dequantised values with the fp32 statistics within the e4m3 step).
"""
from __future__ import annotations

import math
from typing import Dict, Sequence

import numpy as np
import torch

E4M3_MAX = 448.0


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code (ties to even, saturating at +-448) of fp32 values."""
    x = np.clip(np.asarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_decode(codes) -> np.ndarray:
    """fp32 value of e4m3 codes."""
    c = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return c.view(torch.float8_e4m3fn).float().numpy()


def block_summary_fp8(k_block) -> Dict[str, np.ndarray]:
    """FP8 summary of one block k_block [n, d] (values exact in fp32)."""
    k = np.asarray(k_block.detach().float().numpy() if hasattr(k_block, "detach") else k_block, dtype=np.float32)
    n, d = k.shape
    s = np.zeros(d, np.float32)
    for r in range(n):
        s = (s + k[r]).astype(np.float32)
    mean = (s / np.float32(n)).astype(np.float32)
    ss = np.zeros(d, np.float32)
    for r in range(n):
        x = (k[r] - mean).astype(np.float32)
        ss = (ss + (x * x).astype(np.float32)).astype(np.float32)
    sd = np.sqrt((ss / np.float32(n)).astype(np.float32)).astype(np.float32)
    out = {}
    for name, val in (("mu", mean), ("sigma", sd)):
        m = np.float32(np.max(np.abs(val)))
        scl = np.float32(m / np.float32(E4M3_MAX)) if m > 0 else np.float32(1.0)
        code = e4m3_encode((val / scl).astype(np.float32))
        out[name + "_code"] = code
        out[name + "_scale"] = scl
        out[name] = (e4m3_decode(code) * scl).astype(np.float32)
    dev = k.astype(np.float64) - out["mu"].astype(np.float64)
    m = math.sqrt(float((dev * dev).sum(axis=1).max()))
    f = np.float32(m)
    out["max_norm"] = f if float(f) >= m else np.nextafter(f, np.float32(np.inf))
    return out


def summarize_fp8(k, seq_lens: Sequence[int], b: int) -> Dict[str, np.ndarray]:
    """FP8 metadata of a whole cache k [B, Hkv, max_ctx, d] (zero past each
    sequence's last block).  Also returns the dequantised "mu" / "sigma"
    arrays, the form the screen's bound reads."""
    B, Hkv, Tmax, d = k.shape
    nbmax = (Tmax + b - 1) // b
    res = {
        "mu_code": np.zeros((B, Hkv, nbmax, d), np.uint8),
        "sigma_code": np.zeros((B, Hkv, nbmax, d), np.uint8),
        "mu_scale": np.zeros((B, Hkv, nbmax), np.float32),
        "sigma_scale": np.zeros((B, Hkv, nbmax), np.float32),
        "mu": np.zeros((B, Hkv, nbmax, d), np.float32),
        "sigma": np.zeros((B, Hkv, nbmax, d), np.float32),
        "max_norm": np.zeros((B, Hkv, nbmax), np.float32),
    }
    for i, T in enumerate(seq_lens):
        for g in range(Hkv):
            for j in range((T + b - 1) // b):
                blk = block_summary_fp8(k[i, g, j * b:min(T, (j + 1) * b)])
                for name in res:
                    res[name][i, g, j] = blk[name]
    return res
