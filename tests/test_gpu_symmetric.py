"""Symmetric grid on the GPU (zero fixed at 2^(b-1), no zeros array) vs the
oracle: wq_quantize_rtn_sym bit-exact; wq_gemm and wq_gemm_grouped with
zeros = None within the stated tolerance, on every kernel path (M = 1, the
warp-MMA GEMV, the tcgen05 GEMV, the CUDA-core GEMV for odd shapes, the
tcgen05 GEMM), at the BladeLLM block size 64 and at 128 and per row."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from gpu_util import assert_y_close, to_dev_f16, wq

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)


def _gpu_sym(Wh, bits, group):
    c, s, z = wq().wq_quantize_rtn_sym(to_dev_f16(Wh), bits, group)
    assert z is None
    torch.cuda.synchronize()
    return c, s


def _oracle_sym(Wh, bits, group):
    q, s = oracle.quantize_rtn_sym(wq_inputs.f16_bits(Wh), bits, group)
    return oracle.pack(q, bits), s


def _assert_same(Wh, bits, group):
    c, s = _gpu_sym(Wh, bits, group)
    oc, os_ = _oracle_sym(Wh, bits, group)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), os_), "scales differ"
    assert np.array_equal(c.cpu().numpy().view(np.uint32), oc), "codes differ"


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", [32, 64, 128, 0])
def test_sym_quantize_small(bits, group):
    for dist in ("normal", "t4"):
        _assert_same(wq_inputs.weight_f16(40, bits, 37, 384, dist=dist), bits, group)


@pytest.mark.parametrize("bits", BITS)
def test_sym_quantize_long_rows_and_edges(bits):
    _assert_same(wq_inputs.weight_f16(41, bits, 9, 11008, dist="t4"), bits, 0)
    rng = np.random.default_rng(42)
    rows = [np.zeros(64), np.full(64, 1e-8), -np.abs(rng.standard_normal(64)),
            np.abs(rng.standard_normal(64)) * 100, rng.standard_normal(64) * 1e-6,
            rng.integers(-8, 8, 64) * 2.0 ** -5, np.full(64, 65504.0),
            np.concatenate([[-65504.0, 65504.0], rng.standard_normal(62)]),
            np.where(rng.random(64) < 0.5, -0.0, 0.0)]
    _assert_same(np.array(rows).astype(np.float16), bits, 32)


def test_sym_quantize_exhaustive_fp16_sweep():
    from exact import ALL_FINITE_F16
    vals = ALL_FINITE_F16.view(np.float16)
    rows = []
    for a in (1.0, 65504.0, 6e-5, 2e-7, 0.07, 300.0, 2.0 ** -14):
        inside = vals[np.abs(vals.astype(np.float64)) <= a]
        per = 31
        n = (inside.size + per - 1) // per
        pad = np.resize(inside, n * per).reshape(n, per)
        rows.append(np.concatenate([np.full((n, 1), a), pad.astype(np.float64)], 1))
    Wh = np.concatenate(rows).astype(np.float16)
    for bits in BITS:
        _assert_same(Wh, bits, 32)


def _check_gemm(Wh, bits, group, M, seed, grouped=False):
    N, K = Wh.shape
    c, s = _gpu_sym(Wh, bits, group)
    x = wq_inputs.activations_bf16(seed, M, M, K)
    m = wq()
    if grouped:
        (y,) = m.wq_gemm_grouped([(x.cuda(), c, s, None, N, K, group)], bits)
    else:
        y = m.wq_gemm(x.cuda(), c, s, None, bits, group, N, K)
    oc, os_ = _oracle_sym(Wh, bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oracle.sym_zeros(os_, bits), N, K, bits, group)
    assert_y_close(y.float().cpu().numpy(), y_ref, bound, f"sym bits={bits} g={group} M={M} grouped={grouped}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [1, 4, 13, 64, 256])
@pytest.mark.parametrize("group", [64, 128, 0])
def test_sym_gemm(bits, M, group):
    Wh = wq_inputs.weight_f16(43, bits, 300, 1152, dist="t4")
    _check_gemm(Wh, bits, group, M, 43)


@pytest.mark.parametrize("bits", BITS)
def test_sym_gemm_odd_shapes(bits):
    """K not a multiple of 128 (the CUDA-core GEMV at every M)."""
    Wh = wq_inputs.weight_f16(44, bits, 70, 96)
    for M in (1, 5, 40):
        _check_gemm(Wh, bits, 32, M, 44)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [1, 8, 16])
def test_sym_grouped(bits, M):
    Wh = wq_inputs.weight_f16(45, bits, 200, 2048, dist="t4")
    for group in (128, 0):
        _check_gemm(Wh, bits, group, M, 45, grouped=True)


@pytest.mark.parametrize("bits", BITS)
def test_sym_one_hot_exact(bits):
    N, K, group = 64, 1152, 128
    Wh = wq_inputs.weight_f16(46, bits, N, K)
    c, s = _gpu_sym(Wh, bits, group)
    oc, os_ = _oracle_sym(Wh, bits, group)
    w_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oracle.sym_zeros(os_, bits), group)
    m = wq()
    for M in (1, 4, 16):
        for k in (0, 127, 1024, 1151):
            x = torch.zeros(M, K, dtype=torch.bfloat16)
            x[0, k] = -3.0
            y = m.wq_gemm(x.cuda(), c, s, None, bits, group, N, K).cpu()
            assert torch.equal(y[0], (-3.0 * torch.from_numpy(w_ref[:, k])).to(torch.bfloat16)), (M, k)
