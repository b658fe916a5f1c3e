"""Tensor-core decode GEMV (2 <= M <= 16, K a multiple of 128) vs the oracle:
the shapes that reach it -- every group size it accepts, ragged row tiles, K
long enough to be split over a cluster, both batch widths it is built for (up
to 4 and up to 16 rows) -- within the stated tolerance; one-hot activations
exactly; repeated calls bit-identical.  M = 1 cases run alongside, through the
CUDA-core GEMV the dispatch picks for one row."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from gpu_util import assert_y_close, oracle_quantize, to_dev_f16, wq

pytestmark = pytest.mark.gpu


def _run(Wh, x, bits, group):
    N, K = Wh.shape
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K)
    torch.cuda.synchronize()
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, N, K, bits, group)
    return y.float().cpu().numpy(), y_ref, bound


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("group", (32, 64, 128, 256, 0))
def test_groups(bits, group):
    if bits == 3 and group in (32, 64):
        pytest.skip("3-bit with groups below 128 runs on the CUDA-core GEMV")
    N, K = 200, 1024                     # two row tiles, the second ragged
    Wh = wq_inputs.weight_f16(11, bits, N, K, dist="t4")
    for M in (1, 2, 3, 9):
        x = wq_inputs.activations_bf16(11, M, M, K)
        y, yr, b = _run(Wh, x, bits, group)
        assert_y_close(y, yr, b, f"bits={bits} group={group} M={M}")


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("K", (128, 4096, 11008))
def test_split_k(bits, K):
    """One row tile: the launch splits K over a cluster of up to 8 CTAs."""
    N = 128
    Wh = wq_inputs.weight_f16(12, bits, N, K)
    for M in (1, 2, 16):
        x = wq_inputs.activations_bf16(12, M, M, K)
        y, yr, b = _run(Wh, x, bits, 128)
        assert_y_close(y, yr, b, f"bits={bits} K={K} M={M}")


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
def test_one_hot_exact(bits):
    """x = e_k selects column k of W': y equals bf16(w') exactly (s (q - z)
    has at most 19 significant bits, so the fp32 epilogue does not round)."""
    N, K, group = 130, 512, 128
    Wh = wq_inputs.weight_f16(13, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    wq_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
    for k in (0, 1, 7, 63, 127, 128, 200, 511):
        x = torch.zeros(2, K, dtype=torch.bfloat16)     # 2 rows: the tensor-core path
        x[0, k] = 1.0
        x[1, k] = -0.5
        y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
        col = torch.from_numpy(wq_ref[:, k])
        assert torch.equal(y[0], col.to(torch.bfloat16)), f"k={k}"
        assert torch.equal(y[1], (-0.5 * col).to(torch.bfloat16)), f"k={k}"


def test_repeatable():
    N, K, bits, group = 4096, 4096, 3, 128
    Wh = wq_inputs.weight_f16(14, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    x = wq_inputs.activations_bf16(14, 1, 4, K).cuda()       # 4 rows: the tensor-core path
    y0 = m.wq_gemm(x, codes, s, z, bits, group, N, K)
    for _ in range(3):
        assert torch.equal(m.wq_gemm(x, codes, s, z, bits, group, N, K), y0)
    assert m.wq_last_device_error() == m.WQ_OK


def test_large_activations():
    """|x| near 2^62 (the documented range) must not overflow the 2^(64 - b)
    pre-scaled B operand."""
    N, K, bits, group = 128, 256, 2, 128
    Wh = wq_inputs.weight_f16(15, bits, N, K)
    x = (wq_inputs.activations_bf16(15, 1, 2, K).float() * 2.0 ** 60).to(torch.bfloat16)
    y, yr, b = _run(Wh, x, bits, group)
    assert np.all(np.isfinite(y))
    assert_y_close(y, yr, b, "large x")
