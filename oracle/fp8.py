"""FP8 (E4M3) inputs for the oracle: decoding and the exact attention of the decoded inputs.
Plain NumPy. TEST INFRASTRUCTURE ONLY (see the package docstring).

"How does FlashAttention optimize memory and speed via tiling?" (iloveeagents.com), section
"Interview tips", names FP8 among the features of a later FlashAttention version without
defining it. The plainest reading, taken here: Q, K and V arrive as 8-bit E4M3 codes, each
tensor with one fp32 descale factor (the value of a code is its E4M3 value times the factor),
and the method computes the same exact attention (the definition in ``oracle.attention``) of
those values; only the internal arithmetic is allowed lower precision.

E4M3, as defined by the OCP 8-bit floating point specification (and NVIDIA's e4m3 "fn" type):
sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes subnormals
m/8 * 2^-6; the code S.1111.111 is NaN; there are no infinities, so the largest finite value
is 1.75 * 2^8 = 448.
"""

from __future__ import annotations

import numpy as np

from .attention import attention_forward

__all__ = ["e4m3_decode", "attention_forward_fp8", "E4M3_MAX"]

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of uint8 E4M3 codes (NaN for the two NaN codes)."""
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & ((b & 0x7) == 0x7), np.nan, v)


def attention_forward_fp8(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float,
                          scale: float, causal=False, block_rows: int = 512):
    """(O, lse) of exact attention on the decoded inputs: Q = decode(q8) * q_descale, and so on.
    The descale factors are the fp32 values the kernels receive, widened to float64."""
    f = lambda c, s: e4m3_decode(c) * float(np.float32(s))  # noqa: E731
    return attention_forward(f(q8, q_descale), f(k8, k_descale), f(v8, v_descale), scale, causal,
                             block_rows)
