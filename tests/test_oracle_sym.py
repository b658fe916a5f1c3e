"""Pins for the oracle's symmetric grid (no GPU).

The symmetric grid: a = max |w| over the group, scale = the fp16 nearest to
a / (2^(b-1) - 1) (1 if that is 0), zero fixed at 2^(b-1) and not stored,
codes q = clamp(rint(w / scale) + 2^(b-1), 0, 2^b - 1).  Source: "Platform For
AI: BladeLLM model quantization", "Quantization modes > weight_only_quant"
(signed symmetric quantisation is the default) and "block_wise_quant" (one
scale per block of input channels); the scale divisor 2^(b-1) - 1 (the signed
code of +a) is this library's reading.

Each pin checks the oracle against something other than itself: designed
grids with closed-form answers, a brute-force nearest grid point in exact
rational arithmetic, the odd symmetry of round-half-even, and invariants; a
final group plants plausible mistakes and checks the pins reject them.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest
import torch

import wq_inputs
from exact import f16_value, nearest_f16_bits

BITS = (2, 3, 4, 8)


def _designed(bits, group, K, seed):
    rng = np.random.default_rng(seed)
    top = (1 << (bits - 1)) - 1
    z = 1 << (bits - 1)
    N, G = 4, K // group
    cs = rng.integers(-top, top + 1, (N, K))
    s = np.zeros((N, G))
    for n in range(N):
        for j in range(G):
            cs[n, j * group] = top
            cs[n, j * group + 1] = -top
            s[n, j] = 2.0 ** -int(rng.integers(4, 12))
    W = cs * np.repeat(s, group, axis=1)
    Wh = W.astype(np.float16)
    assert np.array_equal(Wh.astype(np.float64), W)
    return Wh, (cs + z).astype(np.uint8), s


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", [32, 64, 128])
def test_sym_designed_grid(orc, bits, group):
    Wh, q, s = _designed(bits, group, 256, seed=7 * bits + group)
    gq, gs = orc.quantize_rtn_sym(wq_inputs.f16_bits(Wh), bits, group)
    assert np.array_equal(gq, q)
    assert np.array_equal(orc.f16_to_f64(gs), s)
    z = orc.sym_zeros(gs, bits)
    assert np.all(orc.f16_to_f64(z) == 2 ** (bits - 1))
    assert np.array_equal(orc.dequant(gq, gs, z, group), Wh.astype(np.float64))


def _brute_sym(wbits, bits):
    qmax = (1 << bits) - 1
    z = 1 << (bits - 1)
    w = [f16_value(int(b)) for b in wbits]
    a = max(abs(v) for v in w)
    sb = nearest_f16_bits(a / (z - 1))
    s = f16_value(sb)
    if s == 0:
        s, sb = Fraction(1), 0x3C00
    codes = []
    for wi in w:
        best = None
        for c in range(qmax + 1):
            key = (abs(wi - s * (c - z)), (c - z) % 2)     # ties: even signed offset
            if best is None or key < best[0]:
                best = (key, c)
        codes.append(best[1])
    return codes, sb


def _groups(bits):
    rng = np.random.default_rng(200 + bits)
    out = []
    for t in range(24):
        kind = t % 6
        if kind == 0:
            g = rng.standard_normal(32) * 0.02
        elif kind == 1:
            g = np.abs(rng.standard_normal(32)) * 3.0       # one sign only
        elif kind == 2:
            g = -np.abs(rng.standard_normal(32)) * 1e-3
        elif kind == 3:
            g = rng.standard_normal(32) * 1e-6               # subnormal scale
        elif kind == 4:
            g = rng.standard_t(4, 32) * 0.02
        else:
            g = rng.integers(-8, 8, 32) * 2.0 ** -5          # exact ties
        out.append(g)
    out.append(np.zeros(32))
    out.append(np.full(32, 1e-8))
    return np.array(out).astype(np.float16)


@pytest.mark.parametrize("bits", BITS)
def test_sym_brute_force(orc, bits):
    W = _groups(bits)
    Wb = wq_inputs.f16_bits(W)
    gq, gs = orc.quantize_rtn_sym(Wb, bits, 32)
    for n in range(W.shape[0]):
        codes, sb = _brute_sym(Wb[n], bits)
        assert gs[n, 0] == sb, n
        assert list(gq[n]) == codes, n


@pytest.mark.parametrize("bits", BITS)
def test_sym_odd_symmetry_and_invariants(orc, bits):
    """rint(-v) = -rint(v), so negating a group mirrors every code about the
    zero (q -> 2^b - q) unless that leaves the code range; every unclamped
    code is within half a step, and +-max|w| lands on the top signed code."""
    N, K, group = 16, 256, 64
    W = wq_inputs.weight_f16(30, bits, N, K, dist="t4")
    Wb, Wn = wq_inputs.f16_bits(W), wq_inputs.f16_bits(-W)
    q, s = orc.quantize_rtn_sym(Wb, bits, group)
    qn, sn = orc.quantize_rtn_sym(Wn, bits, group)
    assert np.array_equal(s, sn)
    z, qmax = 1 << (bits - 1), (1 << bits) - 1
    both = (q >= 1)
    assert np.array_equal(qn[both].astype(int), 2 * z - q[both].astype(int))
    wq = orc.dequant(q, s, orc.sym_zeros(s, bits), group)
    w = W.astype(np.float64)
    sd = np.repeat(orc.f16_to_f64(s), group, axis=1)
    unclamped = (q > 0) & (q < qmax)
    assert np.all(np.abs(w - wq)[unclamped] <= sd[unclamped] / 2)
    for n in range(N):
        for j in range(K // group):
            sl = slice(j * group, (j + 1) * group)
            k = int(np.argmax(np.abs(w[n, sl])))
            exact_scale = abs(w[n, sl][k]) / (z - 1) == sd[n, j * group]
            if exact_scale:
                assert abs(int(q[n, j * group + k]) - z) == z - 1


def test_sym_gemm_exact_small(orc):
    M, N, K, bits, group = 2, 4, 64, 4, 32
    W = wq_inputs.weight_f16(31, 1, N, K)
    x = wq_inputs.activations_bf16(31, 2, M, K)
    q, s = orc.quantize_rtn_sym(wq_inputs.f16_bits(W), bits, group)
    z = orc.sym_zeros(s, bits)
    y, _ = orc.gemm(wq_inputs.bf16_bits(x), orc.pack(q, bits), s, z, N, K, bits, group)
    xv = x.to(torch.float64).numpy()
    for m in range(M):
        for n in range(N):
            ex = sum(Fraction(float(xv[m, k])) * f16_value(int(s[n, k // group])) * (int(q[n, k]) - 8)
                     for k in range(K))
            assert abs(y[m, n] - float(ex)) <= 1e-12 * max(1.0, abs(float(ex)))


def test_sym_pins_reject_planted_mistakes(orc):
    bits = 4
    W = _groups(bits)
    Wb = wq_inputs.f16_bits(W)
    q, s = orc.quantize_rtn_sym(Wb, bits, 32)

    def ok(qq, ss):
        return all(list(qq[n]) == _brute_sym(Wb[n], bits)[0] and ss[n, 0] == _brute_sym(Wb[n], bits)[1]
                   for n in range(W.shape[0]))

    assert ok(q, s)
    w = W.astype(np.float64)
    a = np.abs(w).max(1, keepdims=True)
    # the full-range step 2a / (2^b - 1) instead of a / (2^(b-1) - 1)
    s_wide = orc.f64_to_f16(2 * a / 15)
    sw = np.where(orc.f16_to_f64(s_wide) == 0, 1.0, orc.f16_to_f64(s_wide))
    q_wide = np.clip(np.round(w / sw) + 8, 0, 15).astype(np.uint8)
    assert not ok(q_wide, s_wide)
    # zero one below the middle code
    sd = orc.f16_to_f64(s)
    q_z = np.clip(np.round(w / sd) + 7, 0, 15).astype(np.uint8)
    assert not ok(q_z, s)
    # truncation instead of round-to-nearest
    q_t = np.clip(np.trunc(w / sd) + 8, 0, 15).astype(np.uint8)
    assert not ok(q_t, s)
