"""Pins for the oracle's error-compensating quantiser (OPTQ).

"OPTQ: Accurate Quantization for Generative Pre-trained Transformers"
(reproducibility summary, rows "Experiment Setup" and "Pseudocode") and
"Platform For AI: BladeLLM model quantization" ("Quantization algorithms >
GPTQ") describe the method: quantise the columns of a row in turn and, after
each, adjust the columns not yet quantised through the inverse layer Hessian
so that the layer's output on the calibration activations moves as little as
possible.  These tests hold the oracle to what that fixes, by means other than
its own arithmetic:

* the compensated weights at every step equal the least-squares re-fit of the
  free columns, solved here by ``numpy.linalg.solve``, and each group's grid
  spans the re-fit weights of that group when its first column comes up;
* a diagonal Hessian couples no columns, so the codes, scales and zeros are
  round-to-nearest's bit for bit;
* a power-of-two factor on H changes nothing (it cancels in every step);
* the first column of a row sees no compensation: its code and the first
  group's grid are round-to-nearest's;
* the layer's output error on the calibration rows is well below
  round-to-nearest's.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import wq_inputs as wi


def _case(seed, N, K, S):
    W = wi.f16_bits(wi.weight_f16(seed, 0, N, K))
    X = wi.bf16_bits(wi.calibration_bf16(seed, 0, S, K))
    return W, oracle.hessian(X)


@pytest.mark.parametrize("bits,group", [(3, 32), (4, 0), (2, 64), (8, 32)])
def test_every_step_is_the_least_squares_refit(bits, group):
    """With columns 0..k-1 fixed to their grid values, the weights of the
    free columns k..K-1 minimise (w - w0) H_d (w - w0)^T; column k of that
    minimiser is what the oracle quantises at step k."""
    N, K = 6, 128
    W, H = _case(3, N, K, 384)
    q, s, z, u = oracle.quantize_optq(W, H, bits, group, return_u=True)
    w0 = oracle.f16_to_f64(W)
    wq = oracle.dequant(q, s, z, group)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(K)
    assert np.array_equal(u[:, 0], w0[:, 0])
    scale = np.abs(w0).max()
    g = K if group == 0 else group
    qmax = (1 << bits) - 1
    for k in range(1, K):
        Q, F = np.arange(k), np.arange(k, K)
        refit = w0[:, F] - np.linalg.solve(Hd[np.ix_(F, F)], Hd[np.ix_(F, Q)] @ (wq[:, Q] - w0[:, Q]).T).T
        np.testing.assert_allclose(u[:, k], refit[:, 0], rtol=0, atol=1e-11 * scale, err_msg=f"step {k}")
        if k % g == 0:
            # the group's grid spans the re-fit weights of the whole group at
            # this step (0 included), up to the fp16 rounding of the scale
            v = refit[:, :g]
            span = (np.maximum(v.max(axis=1), 0) - np.minimum(v.min(axis=1), 0)) / qmax
            got = oracle.f16_to_f64(s[:, k // g])
            np.testing.assert_allclose(got, span, rtol=2.0 ** -11, err_msg=f"grid of group {k // g}")


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("group", [32, 64, 0])
def test_diagonal_hessian_gives_round_to_nearest(bits, group):
    N, K = 16, 128
    W = wi.f16_bits(wi.weight_f16(5, 0, N, K))
    H = np.diag(np.random.default_rng(5).uniform(0.1, 10.0, K))
    q, s, z, u = oracle.quantize_optq(W, H, bits, group, return_u=True)
    qr, sr, zr = oracle.quantize_rtn(W, bits, group)
    assert np.array_equal(q, qr)
    assert np.array_equal(s, sr)
    assert np.array_equal(z, zr)
    assert np.array_equal(u, oracle.f16_to_f64(W))


def test_hessian_factor_cancels():
    W, H = _case(6, 8, 96, 256)
    a = oracle.quantize_optq(W, H, 3, 32, return_u=True)
    b = oracle.quantize_optq(W, 4.0 * H, 3, 32, return_u=True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("bits,group", [(3, 32), (4, 0)])
def test_first_column_and_first_grid_are_round_to_nearest(bits, group):
    W, H = _case(7, 32, 128, 256)
    q, s, z = oracle.quantize_optq(W, H, bits, group)
    qr, sr, zr = oracle.quantize_rtn(W, bits, group)
    assert np.array_equal(q[:, 0], qr[:, 0])
    assert np.array_equal(s[:, 0], sr[:, 0])
    assert np.array_equal(z[:, 0], zr[:, 0])
    # later columns do move (the compensation is not a no-op)
    assert (q != qr).mean() > 0.05


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("group", [128, 0])
def test_output_error_below_round_to_nearest(bits, group):
    """trace((W - W') H (W - W')^T), the squared output error on the
    calibration rows, against the same for round-to-nearest codes."""
    N, K = 64, 256
    W, H = _case(4, N, K, 1024)
    w0 = oracle.f16_to_f64(W)

    def err(q, s, z):
        D = w0 - oracle.dequant(q, s, z, group)
        return float(np.einsum("nk,kl,nl->", D, H, D))

    e_optq = err(*oracle.quantize_optq(W, H, bits, group))
    e_rtn = err(*oracle.quantize_rtn(W, bits, group))
    assert e_optq < 0.85 * e_rtn, (e_optq, e_rtn)


def test_codes_within_the_grid_and_packable():
    W, H = _case(8, 16, 96, 256)
    for bits in (2, 3, 4, 8):
        q, s, z = oracle.quantize_optq(W, H, bits, 32)
        assert q.max() <= (1 << bits) - 1
        assert np.array_equal(oracle.unpack(oracle.pack(q, bits), 96, bits), q)


def test_invalid_arguments():
    W, H = _case(9, 4, 64, 128)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_optq(W, H, 5, 32)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_optq(W, H, 4, 48)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_optq(W, H[:32, :32], 4, 32)
    with pytest.raises(oracle.OracleError, match="positive definite"):
        oracle.quantize_optq(W, -np.eye(64), 4, 32)
