"""Dequantisation of the FP8 latent cache format, for the CPU oracle.

TEST INFRASTRUCTURE ONLY (same rule as ``mla_oracle``): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it.

The FP8 cache stores per token:

* the latent cKV as r codes in the OCP FP8 E4M3 format ("e4m3fn"): 1 sign bit,
  4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes the
  subnormals m/8 * 2^-6, the all-ones exponent with all-ones mantissa encodes
  NaN (there is no infinity), so the largest finite value is 1.75 * 2^8 = 448;
* one fp32 scale s_t per token, so that cKV_t = s_t * e4m3(code_t);
* the decoupled RoPE key as bf16 values k_rope'_t stored divided by the token's
  scale, so that k_rope_t = s_t * k_rope'_t (the CUDA path then scales whole
  score columns by s_t).

This module decodes the codes from that definition (bit fields, not a library
cast) and returns the logical cache in float64; the attention itself is
``mla_oracle``'s.
"""

from __future__ import annotations

import numpy as np

__all__ = ["e4m3_value", "e4m3_table", "logical_cache_fp8"]


def e4m3_value(code: int) -> float:
    """The real number an E4M3 code (0..255) stands for; NaN for 0x7F / 0xFF."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """float64 [256]: value of every code."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


_TABLE = e4m3_table()


def logical_cache_fp8(codes_rows: np.ndarray, rope_rows: np.ndarray, scales: np.ndarray):
    """(cKV [L, r], k_rope [L, dr]) in float64 from one sequence's stored rows.

    codes_rows uint8 [L, r], rope_rows (bf16 values as float) [L, dr],
    scales float [L].
    """
    s = np.asarray(scales, dtype=np.float64)[:, None]
    ckv = _TABLE[np.asarray(codes_rows, dtype=np.int64)] * s
    k_rope = np.asarray(rope_rows, dtype=np.float64) * s
    return ckv, k_rope
