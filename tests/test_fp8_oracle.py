"""Pins for the FP8 (e4m3) oracle: rounding against torch's float8_e4m3fn conversion (an
independent implementation of the same round-to-nearest-even) below the saturation threshold,
the saturating behaviour at and above it, the per-tensor scale, and the GEMM of quantised
operands against exact integer arithmetic. CPU only."""
import numpy as np
import torch

import oracle


def test_e4m3_round_matches_torch_float8():
    rng = np.random.default_rng(21)
    # every decade the format covers, subnormals included, plus exact ties
    mags = np.exp2(rng.uniform(-12, np.log2(460), size=200000))
    v = (mags * rng.choice([-1.0, 1.0], size=mags.size)).astype(np.float32)
    grid = torch.arange(0, 256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    grid = grid[np.isfinite(grid) & (np.abs(grid) <= 448)]
    pos = np.unique(np.abs(grid))
    ties = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)  # midpoints between neighbours
    v = np.concatenate([v, ties[ties < 460], -ties[ties < 460], grid.astype(np.float32)])
    ref = torch.tensor(v).to(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_round(v)
    assert np.array_equal(got, ref.astype(np.float64))


def test_e4m3_saturates_and_keeps_zero():
    big = np.array([464.0, 500.0, 1e6, -464.0, -3e4], np.float32)
    assert np.array_equal(oracle.e4m3_round(big), np.array([448, 448, 448, -448, -448.0]))
    assert np.array_equal(oracle.e4m3_round(np.array([0.0, 2.0 ** -11, -2.0 ** -11])),
                          np.zeros(3))


def test_quantize_scale_and_error_bound():
    rng = np.random.default_rng(3)
    x = (rng.normal(size=(64, 96)) * 3.0).astype(np.float32)
    q, amax, d = oracle.quantize_e4m3(x)
    assert amax == float(np.max(np.abs(x)))
    assert np.max(np.abs(q)) == 448.0  # the largest magnitude lands on the top of the grid
    assert d == float(np.float32(amax) / np.float32(448.0))
    # relative rounding error of a normal e4m3 value is at most 2^-4
    deq = q * d
    big = np.abs(x) > amax * 2.0 ** -6 * 2  # comfortably in the normal range
    assert np.max(np.abs(deq[big] - x[big]) / np.abs(x[big])) <= 2.0 ** -4 * 1.0001
    z, amax0, d0 = oracle.quantize_e4m3(np.zeros(5))
    assert amax0 == 0.0 and d0 == 1.0 and not np.any(z)


def test_gemm_fp8_is_exact_integer_arithmetic():
    """e4m3 values are integer multiples of 2^-9, so (2^9 qa)(2^9 qb)^T is an exact int64
    matrix product; the fp64 GEMM of the oracle must reproduce it exactly (products and sums
    of these values are exact in fp64 for K up to 2^16)."""
    rng = np.random.default_rng(9)
    qa, _, _ = oracle.quantize_e4m3(rng.normal(size=(40, 256)))
    qb, _, _ = oracle.quantize_e4m3(rng.normal(size=(24, 256)))
    ia = np.round(qa * 512).astype(np.int64)
    ib = np.round(qb * 512).astype(np.int64)
    exact = (ia @ ib.T).astype(np.float64) / 512.0 / 512.0
    assert np.array_equal(oracle.gemm_fp8(qa, 1.0, qb, 1.0), exact)
    assert np.allclose(oracle.gemm_fp8(qa, 0.5, qb, 3.0), exact * 1.5, rtol=0, atol=0)
