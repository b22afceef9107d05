"""fp64 oracle for the FP8 (e4m3) path: per-tensor quantisation and the GEMM of quantised
operands.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources: the page "把大模型训练“摁”到规模化：NVIDIA Megatron-LM / Megatron Core 上手与理解"
(vampireachao.github.io), section 0, lists FP8 among Megatron Core's mixed precisions; the
trdm.cn page's inference section enables it with --enable-fp8. The pages give no format or
scaling recipe. Readings (also in the design notes):
  * format e4m3 ("fn": 4 exponent bits with bias 7, 3 mantissa bits, no infinities): normal
    values 1.m * 2^(e-7) for e = 1..15 except the all-ones pattern, so the largest finite
    value is 1.75 * 2^8 = 448; subnormals m * 2^-9, m = 1..7;
  * per-tensor current scaling: amax = max |x|, s = 448 / amax (1 if amax = 0), q = e4m3(x * s)
    rounded to nearest, ties to even, saturating at +-448; dequantisation factor amax / 448;
  * the GPU forms x * s and the scale in fp32 before rounding, so the oracle does too: the
    rounding decision is taken on the same fp32 number.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_round(v):
    """Nearest e4m3 value (ties to even, saturating at +-448) of each entry of v, as float64.
    Written from the format: for |v| in [2^e, 2^(e+1)) with e >= -6 the spacing is 2^(e-3);
    below 2^-6 (subnormals) it is 2^-9."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    step = np.exp2(e - 3.0)
    q = np.round(a / step) * step  # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(a > 0, np.sign(v) * q, 0.0)


def quantize_e4m3(x):
    """Per-tensor quantisation of x (any shape). Returns (q as float64 e4m3 values, amax,
    dequantisation factor): q = e4m3(fp32(x) * s), s = fp32(448 / amax)."""
    x32 = np.asarray(x, np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    s = np.float32(448.0) / amax if amax > 0 else np.float32(1.0)
    scaled = (x32 * s).astype(np.float32)  # one fp32 rounding, as on the GPU
    q = e4m3_round(scaled)
    d = np.float32(amax) / np.float32(448.0) if amax > 0 else np.float32(1.0)
    return q, float(amax), float(d)


def gemm_fp8(qa, da, qb, db):
    """C = (qa @ qb^T) * da * db in float64: qa [M, K], qb [N, K] e4m3 values (exact in fp64),
    da, db the dequantisation factors."""
    return (np.asarray(qa, np.float64) @ np.asarray(qb, np.float64).T) * (float(da) * float(db))
