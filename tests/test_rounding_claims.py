"""CPU pins for the arithmetic claims the CUDA quantiser relies on.

The library computes codes and zeros as ``rint(a / s)`` with an IEEE fp32
division (correctly rounded) and the scale as one fp64 division rounded once to
fp16.  Both are claimed to equal exact rational rounding for every input the
grid can produce.  These tests check the claims directly, with numpy's IEEE
float32/float64 arithmetic standing in for the device's ``div.rn`` and integer
arithmetic standing in for the exact result.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from exact import ALL_FINITE_F16, f16_value, nearest_f16_bits


def _exact_rint_ratio(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Round-half-even of A/B for integer arrays, B > 0."""
    q = np.floor_divide(A, B)
    r = A - q * B                 # 0 <= r < B
    twice = 2 * r
    up = (twice > B) | ((twice == B) & (q % 2 == 1))
    return q + up


def test_fp32_division_rint_is_exact_over_all_fp16():
    w = ALL_FINITE_F16.view(np.float16)
    W_int = (w.astype(np.float64) * 2.0 ** 24).astype(np.int64)       # exact: fp16 = n * 2^-24
    rng = np.random.default_rng(0)
    sbits = np.unique(np.concatenate([
        np.arange(1, 64, dtype=np.uint16),                          # subnormal scales
        np.arange(0x0400, 0x7C00, 97, dtype=np.uint16),              # spread over normals
        rng.integers(0x0001, 0x7C00, 200).astype(np.uint16),
        np.array([0x3C00, 0x2E66, 0x1A36, 0x7BFF, 0x0400, 0x03FF], dtype=np.uint16)]))
    w32 = w.astype(np.float32)
    for sb in sbits:
        s = np.array([sb], np.uint16).view(np.float16)[0]
        S_int = int(float(s) * 2.0 ** 24)
        exact = _exact_rint_ratio(W_int, np.int64(S_int))
        keep = np.abs(W_int) < 2048 * S_int          # codes clamp beyond this either way
        f32 = np.rint(w32 / np.float32(s)).astype(np.int64)
        f64 = np.rint(w.astype(np.float64) / float(s)).astype(np.int64)
        assert np.array_equal(f32[keep], exact[keep]), hex(sb)
        assert np.array_equal(f64[keep], exact[keep]), hex(sb)


def test_fp64_scale_rounds_once_to_nearest_fp16():
    rng = np.random.default_rng(1)
    lo = -np.abs(rng.standard_normal(4000) * 10.0 ** rng.integers(-7, 4, 4000)).astype(np.float16)
    hi = np.abs(rng.standard_normal(4000) * 10.0 ** rng.integers(-7, 4, 4000)).astype(np.float16)
    for qmax in (3, 7, 15, 255):
        d = (hi.astype(np.float64) - lo.astype(np.float64)) / qmax        # fp64 path
        got = d.astype(np.float16).view(np.uint16)                          # one RNE to fp16
        for i in range(0, 4000, 7):
            ex = (f16_value(int(hi.view(np.uint16)[i])) - f16_value(int(lo.view(np.uint16)[i]))) / qmax
            assert got[i] == nearest_f16_bits(ex)
