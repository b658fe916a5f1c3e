"""Pins for the CPU oracle (no GPU).

The oracle must be right before anything is compared with it, so each of its
functions is checked against something other than itself:

* format conversions: exhaustive decode vs numpy/torch casts, RNE midpoints and
  random values vs exact rational search;
* quantiser: closed-form designed grids (the stored parameters and codes must
  come back exactly), brute-force nearest grid point in exact rationals, the
  nearest-fp16 scale by search, invariants of the min-max grid;
* packing: hand-derived words (tests/golden/packing.txt), round trips;
* matmul: exact rational sums on tiny inputs, one-hot and zero inputs,
  permutation invariance.

A final group plants plausible mistakes into oracle outputs and checks that the
pins reject them.

Sources: "OPTQ: Accurate Quantization for Generative Pre-trained Transformers"
(reproducibility summary, "Experiment Setup": per-row asymmetric min-max grid);
"Platform For AI: BladeLLM model quantization" ("block_wise_quant" groups,
"Quantization algorithms > MinMax" round-to-nearest); "[Feature Request] 4bit
and 2bit and 1bit quantization support" (codes packed several per word).
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import wq_inputs
from exact import ALL_FINITE_F16, f16_value, nearest_f16_bits, round_half_even

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = (2, 3, 4, 8)


# --------------------------------------------------------------------- formats
def test_f16_decode_exhaustive(orc):
    allb = np.arange(1 << 16, dtype=np.uint16)
    got = orc.f16_to_f64(allb)
    ref = allb.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))
    assert np.all(np.isinf(got[np.isinf(ref)])) and np.all(np.isnan(got[np.isnan(ref)]))


def test_bf16_decode_exhaustive(orc):
    allb = np.arange(1 << 16, dtype=np.uint16)
    got = orc.bf16_to_f64(allb)
    ref = torch.from_numpy(allb.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.all(np.isnan(got[np.isnan(ref)]))


def test_f16_round_midpoints_and_random(orc):
    pos = np.arange(0, 0x7C00, dtype=np.uint16)
    v = pos.view(np.float16).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2          # exact in fp64: every tie case
    rng = np.random.default_rng(1)
    rnd = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
                          [65504.0, 65519.0, 65519.999, 65520.0, 70000.0, 2.0 ** -25,
                           2.0 ** -25 * 1.0000001, 2.0 ** -26, 3 * 2.0 ** -26, 0.0]])
    d = np.concatenate([mids, -mids, rnd, -rnd])
    got = orc.f64_to_f16(d)
    ref = d.astype(np.float16).view(np.uint16)      # numpy: one RNE rounding
    assert np.array_equal(got, ref)


def test_f16_round_exact_search(orc):
    rng = np.random.default_rng(2)
    vals = [Fraction(int(a), int(b)) for a, b in zip(rng.integers(1, 1 << 40, 300),
                                                     rng.integers(1, 1 << 30, 300))]
    vals += [f16_value(0x3C00) + Fraction(1, 2048), f16_value(0x3C01) + Fraction(1, 2048)]
    got = orc.f64_to_f16(np.array([float(v) for v in vals]))
    for v, g in zip(vals, got):
        if float(v) == v:   # representable in fp64: the exact search applies directly
            assert g == nearest_f16_bits(v), v


def test_bf16_round_vs_torch(orc):
    rng = np.random.default_rng(3)
    f = rng.standard_normal(50000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 50000).astype(np.float32)
    pos = np.arange(0, 0x7F80, dtype=np.uint16)
    bv = torch.from_numpy(pos.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    mids = ((bv[:-1] + bv[1:]) / 2).astype(np.float32)     # bf16 midpoints are fp32 values
    d = np.concatenate([f, mids, -mids]).astype(np.float32)
    got = orc.f64_to_bf16(d.astype(np.float64))
    ref = torch.from_numpy(d).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------- packing
def _golden_packing():
    rows = []
    with open(os.path.join(GOLDEN, "packing.txt")) as fh:
        for line in fh:
            if not line.strip() or line.startswith("#"):
                continue
            b, codes, words, _ = [p.strip() for p in line.split("|")]
            rows.append((int(b), [int(c) for c in codes.split()], [int(w, 16) for w in words.split()]))
    return rows


@pytest.mark.parametrize("case", range(5))
def test_pack_golden(orc, case):
    bits, codes, words = _golden_packing()[case]
    K = 32 * ((len(codes) + 31) // 32)
    q = np.zeros((1, K), np.uint8)
    q[0, :len(codes)] = codes
    w = orc.pack(q, bits)
    assert list(w[0, :len(words)]) == words
    assert not w[0, len(words):].any()
    assert np.array_equal(orc.unpack(w, K, bits), q)


@pytest.mark.parametrize("bits", BITS)
def test_pack_roundtrip(orc, bits):
    rng = np.random.default_rng(bits)
    K = 32 * 7
    q = rng.integers(0, 1 << bits, (5, K)).astype(np.uint8)
    w = orc.pack(q, bits)
    assert w.shape == (5, K * bits // 32)
    assert np.array_equal(orc.unpack(w, K, bits), q)
    # unpack(pack(.)) is the identity on arbitrary words, too
    words = rng.integers(0, 1 << 32, (3, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(orc.pack(orc.unpack(words, K, bits), bits), words)


# --------------------------------------------------------------------- quantiser
def _designed(bits, group, K, seed):
    """Weights that lie exactly on a grid with power-of-two scale and integer
    zero, both ends of the code range used in every group."""
    rng = np.random.default_rng(seed)
    qmax = (1 << bits) - 1
    N = 4
    G = K // group
    q = rng.integers(0, qmax + 1, (N, K))
    s = np.zeros((N, G))
    z = np.zeros((N, G), dtype=np.int64)
    W = np.zeros((N, K))
    for n in range(N):
        for j in range(G):
            sl = slice(j * group, (j + 1) * group)
            q[n, j * group] = 0
            q[n, j * group + 1] = qmax
            s[n, j] = 2.0 ** -int(rng.integers(4, 12))
            z[n, j] = rng.integers(0, qmax + 1)
            W[n, sl] = s[n, j] * (q[n, sl] - z[n, j])
    Wh = W.astype(np.float16)
    assert np.array_equal(Wh.astype(np.float64), W)     # exactly representable
    return Wh, q, s, z


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", [32, 128])
def test_quantize_designed_grid(orc, bits, group):
    Wh, q, s, z = _designed(bits, group, 256, seed=10 * bits + group)
    gq, gs, gz = orc.quantize_rtn(wq_inputs.f16_bits(Wh), bits, group)
    assert np.array_equal(gq, q)
    assert np.array_equal(orc.f16_to_f64(gs), s)
    assert np.array_equal(orc.f16_to_f64(gz), z.astype(np.float64))
    assert np.array_equal(orc.dequant(gq, gs, gz, group), Wh.astype(np.float64))


def _brute_group(wbits, bits):
    """Exact-rational restatement by search: nearest fp16 to the min-max step,
    nearest integer zero, nearest grid point per weight (ties: even offset)."""
    qmax = (1 << bits) - 1
    w = [f16_value(int(b)) for b in wbits]
    lo, hi = min([Fraction(0)] + w), max([Fraction(0)] + w)
    sb = nearest_f16_bits((hi - lo) / qmax)
    s = f16_value(sb)
    if s == 0:
        s, sb, z = Fraction(1), 0x3C00, 0
    else:
        z = round_half_even(-lo / s)
    codes = []
    for wi in w:
        best = None
        for c in range(qmax + 1):
            d = abs(wi - s * (c - z))
            key = (d, (c - z) % 2)      # prefer the even offset on a tie
            if best is None or key < best[0]:
                best = (key, c)
        codes.append(best[1])
    return codes, sb, z


@pytest.mark.parametrize("bits", BITS)
def test_quantize_brute_force(orc, bits):
    rng = np.random.default_rng(100 + bits)
    groups = []
    for t in range(24):
        kind = t % 6
        if kind == 0:
            g = rng.standard_normal(32) * 0.02
        elif kind == 1:
            g = np.abs(rng.standard_normal(32)) * 3.0          # same sign: R1 matters
        elif kind == 2:
            g = -np.abs(rng.standard_normal(32)) * 1e-3
        elif kind == 3:
            g = rng.standard_normal(32) * 1e-6                  # subnormal scale
        elif kind == 4:
            g = rng.standard_t(4, 32) * 0.02
        else:
            g = rng.integers(-8, 8, 32) * 2.0 ** -5             # many exact ties
        groups.append(g)
    groups.append(np.zeros(32))                                 # degenerate
    groups.append(np.full(32, 1e-8))                            # scale underflows
    W = np.array(groups).astype(np.float16)
    Wb = wq_inputs.f16_bits(W)
    gq, gs, gz = orc.quantize_rtn(Wb, bits, 32)
    for n in range(W.shape[0]):
        codes, sb, z = _brute_group(Wb[n], bits)
        assert gs[n, 0] == sb, n
        assert orc.f16_to_f64(gz[n:n + 1, :1])[0, 0] == z, n
        assert gz[n, 0] & 0x8000 == 0
        assert list(gq[n]) == codes, n


def test_quantize_ties_exact(orc):
    # Weights sitting exactly halfway between two grid points: with scale 1/4
    # (range [-1, 2.75] at 4 bits) w = (n + 1/2)/4 must round to the even offset.
    qmax = 15
    base = np.array([-1.0, 2.75] + [(n + 0.5) / 4 for n in range(-4, 10)] + [0.0] * 16)
    W = base[None, :].astype(np.float16)
    gq, gs, gz = orc.quantize_rtn(wq_inputs.f16_bits(W), 4, 32)
    assert orc.f16_to_f64(gs)[0, 0] == 0.25 and orc.f16_to_f64(gz)[0, 0] == 4
    for k in range(2, 16):
        t = base[k] / 0.25              # n + 1/2
        n = int(np.floor(t))
        even = n if n % 2 == 0 else n + 1
        assert gq[0, k] == min(max(even + 4, 0), qmax)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", [0, 64])
def test_quantize_invariants(orc, bits, group):
    N, K = 16, 256
    W = wq_inputs.weight_f16(5, bits, N, K, dist="t4")
    Wb = wq_inputs.f16_bits(W)
    q, s, z = orc.quantize_rtn(Wb, bits, group)
    g = K if group == 0 else group
    qmax = (1 << bits) - 1
    assert q.max() <= qmax
    sd, zd = orc.f16_to_f64(s), orc.f16_to_f64(z)
    assert np.all(zd == np.round(zd)) and np.all(zd >= 0)
    wq = orc.dequant(q, s, z, group)
    w = W.astype(np.float64)
    for n in range(N):
        for j in range(K // g):
            sl = slice(j * g, (j + 1) * g)
            sc = sd[n, j]
            ulp = 2.0 ** (np.floor(np.log2(sc)) - 10)
            err = np.abs(w[n, sl] - wq[n, sl])
            unclamped = (q[n, sl] > 0) & (q[n, sl] < qmax)
            assert np.all(err[unclamped] <= sc / 2)
            assert np.all(err <= sc / 2 + qmax * ulp / 2)
            # the group's minimum (<= 0 here) is reproduced by code 0
            kmin = int(np.argmin(w[n, sl]))
            if w[n, sl][kmin] <= 0:
                assert q[n, j * g + kmin] == 0


def test_quantize_per_row_equals_group_k(orc):
    W = wq_inputs.f16_bits(wq_inputs.weight_f16(7, 0, 8, 320))
    a = orc.quantize_rtn(W, 3, 0)
    b = orc.quantize_rtn(W, 3, 320)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_quantize_rejects_bad_args(orc):
    W = np.zeros((2, 64), np.uint16)
    for bits, group in [(5, 32), (1, 32), (4, 48), (4, 16), (4, -32)]:
        with pytest.raises(orc.OracleError):
            orc.quantize_rtn(W, bits, group)
    with pytest.raises(orc.OracleError):
        orc.quantize_rtn(np.zeros((2, 40), np.uint16), 4, 0)


# --------------------------------------------------------------------- matmul
def test_gemm_exact_small(orc):
    rng = np.random.default_rng(11)
    M, N, K, bits, group = 3, 5, 64, 3, 32
    W = wq_inputs.weight_f16(11, 1, N, K)
    x = wq_inputs.activations_bf16(11, 2, M, K)
    xb = wq_inputs.bf16_bits(x)
    q, s, z = orc.quantize_rtn(wq_inputs.f16_bits(W), bits, group)
    words = orc.pack(q, bits)
    y, bnd = orc.gemm(xb, words, s, z, N, K, bits, group)
    xv = x.to(torch.float64).numpy()
    sv = [[f16_value(int(v)) for v in row] for row in s]
    zv = [[f16_value(int(v)) for v in row] for row in z]
    for m in range(M):
        for n in range(N):
            ex = sum(Fraction(float(xv[m, k])) * sv[n][k // group] * (int(q[n, k]) - zv[n][k // group])
                     for k in range(K))
            eb = sum(abs(Fraction(float(xv[m, k])) * sv[n][k // group] * (int(q[n, k]) - zv[n][k // group]))
                     for k in range(K))
            tol = float(eb) * K * 2.0 ** -52
            assert abs(y[m, n] - float(ex)) <= tol
            assert abs(bnd[m, n] - float(eb)) <= tol
    # a subset of columns gives the same numbers
    y2, b2 = orc.gemm(xb, words, s, z, N, K, bits, group, cols=[4, 0, 2])
    assert np.array_equal(y2, y[:, [4, 0, 2]]) and np.array_equal(b2, bnd[:, [4, 0, 2]])


@pytest.mark.parametrize("bits", BITS)
def test_gemm_one_hot_and_zero(orc, bits):
    N, K, group = 6, 128, 64
    W = wq_inputs.f16_bits(wq_inputs.weight_f16(12, bits, N, K))
    q, s, z = orc.quantize_rtn(W, bits, group)
    words = orc.pack(q, bits)
    wq = orc.dequant(q, s, z, group)
    for k in (0, 31, 64, 127):
        x = torch.zeros(1, K, dtype=torch.bfloat16)
        x[0, k] = 1.0
        y, _ = orc.gemm(wq_inputs.bf16_bits(x), words, s, z, N, K, bits, group)
        assert np.array_equal(y[0], wq[:, k])
    y, b = orc.gemm(np.zeros((2, K), np.uint16), words, s, z, N, K, bits, group)
    assert not y.any() and not b.any()


def test_gemm_block_permutation(orc):
    N, K, group, bits = 4, 256, 64, 4
    W = wq_inputs.weight_f16(13, 0, N, K)
    x = wq_inputs.activations_bf16(13, 1, 2, K)
    perm = np.concatenate([np.arange(j * group, (j + 1) * group) for j in (2, 0, 3, 1)])
    ys = []
    for p in (np.arange(K), perm):
        q, s, z = orc.quantize_rtn(wq_inputs.f16_bits(W[:, p]), bits, group)
        y, b = orc.gemm(wq_inputs.bf16_bits(x[:, p]), orc.pack(q, bits), s, z, N, K, bits, group)
        ys.append((y, b))
    assert np.allclose(ys[0][0], ys[1][0], rtol=0, atol=1e-12 * ys[0][1].max())


# --------------------------------------------------------------------- planted mistakes
def _brute_ok(orc, Wb, bits, q, s, z):
    for n in range(Wb.shape[0]):
        codes, sb, zz = _brute_group(Wb[n], bits)
        if s[n, 0] != sb or orc.f16_to_f64(z[n:n + 1, :1])[0, 0] != zz or list(q[n]) != codes:
            return False
    return True


def test_pins_reject_planted_mistakes(orc):
    bits = 4
    W = np.array([np.random.default_rng(20 + i).standard_normal(32) * 0.02 for i in range(300)])
    Wb = wq_inputs.f16_bits(W.astype(np.float16))
    q, s, z = orc.quantize_rtn(Wb, bits, 32)
    assert _brute_ok(orc, Wb, bits, q, s, z)
    # off-by-one zero
    z_bad = orc.f64_to_f16(orc.f16_to_f64(z) + 1)
    assert not _brute_ok(orc, Wb, bits, q, s, z_bad)
    # truncation instead of round-to-nearest
    s_d, z_d = orc.f16_to_f64(s), orc.f16_to_f64(z)
    w = W.astype(np.float16).astype(np.float64)
    q_trunc = np.clip(np.trunc(w / s_d) + z_d, 0, 15).astype(np.uint8)
    assert not _brute_ok(orc, Wb, bits, q_trunc, s, z)
    # unrounded (fp64) scale used for the codes
    lo = np.minimum(w.min(1, keepdims=True), 0)
    hi = np.maximum(w.max(1, keepdims=True), 0)
    s64 = (hi - lo) / 15
    q_s64 = np.clip(np.round(w / s64) + np.round(-lo / s64), 0, 15).astype(np.uint8)
    assert not _brute_ok(orc, Wb, bits, q_s64, s, z)
    # a transposed / dropped term in the matmul is caught by the exact sum
    N, K, group = 3, 64, 32
    Wt = wq_inputs.weight_f16(21, 0, N, K)
    qq, ss, zz = orc.quantize_rtn(wq_inputs.f16_bits(Wt), 3, group)
    x = wq_inputs.activations_bf16(21, 1, 1, K)
    y, _ = orc.gemm(wq_inputs.bf16_bits(x), orc.pack(qq, 3), ss, zz, N, K, 3, group)
    wq = orc.dequant(qq, ss, zz, group)
    xv = x.to(torch.float64).numpy()
    assert np.allclose(y[0], wq @ xv[0], rtol=1e-12, atol=1e-15)
    assert not np.allclose(y[0], wq[:, :-1] @ xv[0, :-1], rtol=1e-9, atol=0)
