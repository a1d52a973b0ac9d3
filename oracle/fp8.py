"""FP8 (e4m3) KV cache: decoding of the stored bytes (test oracle; see package doc).

Why it exists: decode attention is bound by the bytes of K and V it streams,
and storing the cache in 8-bit floats halves them (blog post "Prefill vs.
Decode GPU Utilization Imbalance", section "Quantization and compression as a
lever on both the bandwidth and capacity problem").  The attention itself is
unchanged: the oracle decodes every stored byte exactly to float64, multiplies
by its kv head's scale, and runs the same float64 decode attention
(``attention.attend_decode``) on the result.

e4m3 (the "E4M3" 8-bit float of the OCP FP8 formats): bit 7 = sign s, bits 6..3
= exponent e (bias 7), bits 2..0 = mantissa m.
  e in 1..15:  (-1)^s * 2^(e-7) * (1 + m/8), except e = 15, m = 7 (NaN);
  e = 0:       (-1)^s * 2^-6 * (m/8)          (subnormals and zero).
There is no infinity; the largest finite magnitude is 2^8 * 1.75 = 448.

Reading taken where the sources are silent: one fp32 scale per kv head for K
and one for V (dequantised value = scale[kv head] * e4m3 value); the prefill
requests keep reading the bf16 cache (the FP8 cache serves the decode branch).
"""
from __future__ import annotations

import numpy as np


def e4m3_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of each e4m3 byte (uint8) as float64; NaN for the NaN codes."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 0x7
    sign = np.where(s == 1, -1.0, 1.0)
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    out = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, out)


def dequant_pool(pool_u8: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[num_blocks, Hkv, 16, d] e4m3 bytes -> float64 values scale[kv head] * e4m3."""
    vals = e4m3_to_f64(pool_u8)
    sc = np.asarray(scales, dtype=np.float32).astype(np.float64)
    return vals * sc[None, :, None, None]
