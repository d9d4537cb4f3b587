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

Every statistic is the definition evaluated in float64 from the exact inputs:
the mean and the population standard deviation of the block's rows per
coordinate, the scale as the fp32 value nearest to (largest magnitude) / 448,
the code as the e4m3 value nearest to the float64 quotient (statistic /
scale), ties to the even code, saturating at +-448 (the encoder below follows
the e4m3 format's definition: 4 exponent bits with bias 7, 3 fraction bits,
subnormal step 2^-9).  The dequantised centroid is code value x scale, exact
in float64, and M is the largest distance of a row from it, rounded up to
fp32.

Parity status: pinned by tests/test_oracle_fp8_pins.py (the e4m3 rounding
against a brute-force nearest-value search over all 256 codes, in fp32 and at
float64 points next to every rounding boundary; closed forms of the scale and
of a constant block; the statistics against numpy's mean and population std;
the strict bound by brute force; the dequantised values within half an e4m3
step of the exact statistics).
"""
from __future__ import annotations

import math
from typing import Dict, Sequence

import numpy as np
import torch

E4M3_MAX = 448.0


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code of each value (float64 or narrower, taken exactly):
    ties to the even code, saturating at +-448; the sign bit follows the
    value's sign (a negative value that rounds to zero gives -0, code 0x80)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # normal range: |x| = f 2^e with f in [1, 2), kept to 3 fraction bits
    f, ex = np.frexp(np.where(a > 0, a, 1.0))   # a = f 2^ex, f in [0.5, 1)
    e = ex - 1
    q = np.rint(f * 16.0)                        # (1 + m/8) * 8 rounded, in [8, 16]
    carry = q == 16.0
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 8.0, q)
    normal_code = (e + 7) * 8 + (q - 8)
    # below 2^-6: multiples of 2^-9 (code k = k 2^-9; k = 8 is 2^-6, code 0x08)
    sub_code = np.rint(a * 512.0)
    code = np.where(a < 2.0 ** -6, sub_code, normal_code).astype(np.int64)
    code = np.minimum(code, 0x7E)
    sign = np.signbit(x).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """fp32 value of e4m3 codes."""
    c = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return c.view(torch.float8_e4m3fn).float().numpy()


def fp32_nearest(x: float) -> np.float32:
    """The fp32 value nearest to x (ties to even)."""
    return np.float32(x)


def block_summary_fp8(k_block) -> Dict[str, np.ndarray]:
    """FP8 summary of one block k_block [n, d] (values exact in fp32)."""
    k = np.asarray(k_block.detach().float().numpy() if hasattr(k_block, "detach") else k_block, dtype=np.float64)
    n, d = k.shape
    mean = k.sum(axis=0) / n
    sd = np.sqrt(((k - mean) ** 2).sum(axis=0) / n)
    out = {}
    for name, val in (("mu", mean), ("sigma", sd)):
        m = float(np.max(np.abs(val)))
        scl = fp32_nearest(m / E4M3_MAX) if m > 0 else np.float32(1.0)
        code = e4m3_encode(val / float(scl))
        out[name + "_code"] = code
        out[name + "_scale"] = scl
        out[name] = e4m3_decode(code).astype(np.float64) * float(scl)
    dev = k - out["mu"]
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
        "mu": np.zeros((B, Hkv, nbmax, d), np.float64),
        "sigma": np.zeros((B, Hkv, nbmax, d), np.float64),
        "max_norm": np.zeros((B, Hkv, nbmax), np.float32),
    }
    for i, T in enumerate(seq_lens):
        for g in range(Hkv):
            for j in range((T + b - 1) // b):
                blk = block_summary_fp8(k[i, g, j * b:min(T, (j + 1) * b)])
                for name in res:
                    res[name][i, g, j] = blk[name]
    return res
