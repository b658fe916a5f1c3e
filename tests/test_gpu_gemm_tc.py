"""Tensor-core GEMM (M > 16) vs the oracle: y within the stated tolerance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from gpu_util import assert_y_close, cached_weight, oracle_quantize, to_dev_f16, wq

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)


def _run(Wh, x, bits, group):
    N, K = Wh.shape
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K)
    torch.cuda.synchronize()
    assert m.wq_last_device_error() == m.WQ_OK
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, N, K, bits, group)
    return y.float().cpu().numpy(), y_ref, bound


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M,N,K,group", [
    (17, 256, 128, 128), (64, 300, 384, 32), (256, 256, 256, 0), (257, 200, 640, 128),
    (520, 513, 384, 64),
    # groups spanning several K-step pairs, and one that splits a pair
    (96, 384, 1024, 256), (33, 130, 768, 384), (48, 200, 384, 96),
    # few output tiles and a long K: split-K over a cluster of CTAs
    (300, 520, 4096, 128), (40, 256, 2048, 0)])
def test_tc_small(bits, M, N, K, group):
    Wh = wq_inputs.weight_f16(8, bits, N, K)
    x = wq_inputs.activations_bf16(8, M, M, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, f"bits={bits} M={M} N={N} K={K} g={group}")


def test_tc_k_not_multiple_of_128_uses_gemv_chunks():
    N, K, M, bits, group = 70, 4160, 40, 4, 32
    Wh = wq_inputs.weight_f16(9, 0, N, K)
    x = wq_inputs.activations_bf16(9, 1, M, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, "K=4160 M=40")


@pytest.mark.parametrize("bits", BITS)
def test_tc_one_hot_exact(bits):
    N, K, M, group = 256, 256, 32, 128
    Wh = wq_inputs.weight_f16(10, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    wq_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    ks = [(7 * i) % K for i in range(M)]
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
    for i, k in enumerate(ks):
        assert torch.equal(y[i], torch.from_numpy(wq_ref[:, k]).to(torch.bfloat16)), (i, k)


@pytest.mark.parametrize("cfg,linear,M", [
    ("llama13b_prefill_4b_g128", 0, 2048), ("llama13b_prefill_4b_g128", 1, 2048),
    ("llama7b_stack32_4b_g128", 0, 64), ("llama7b_stack32_4b_g128", 6, 64)])
def test_tc_full_size_sampled(cfg, linear, M):
    w = wq_inputs.WORKLOADS[cfg]
    name, N, K = w["linears"][linear]
    bits, group = w["bits"], w["group"]
    Wh = cached_weight(0, linear, N, K, w["dist"])
    x = wq_inputs.activations_bf16(0, 200 + linear, M, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).float().cpu().numpy()
    assert m.wq_last_device_error() == m.WQ_OK
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(8).integers(0, N, 62)]))
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(9).integers(0, M, 30)]))
    oc, os_, oz = oracle_quantize(Wh[cols], bits, group)
    xs = x[torch.from_numpy(rows)]
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(xs), oc, os_, oz, len(cols), K, bits, group)
    assert_y_close(y[np.ix_(rows, cols)], y_ref, bound, f"{cfg}/{name} M={M}")


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 0)])
def test_tc_whole_waves_then_split_rest(bits, group):
    """152 tiles of 256 x 256 on 148 SMs: one launch of 148 whole tiles, then
    the 4 left over with K split over a cluster.  Rows of the first and the
    last row of tiles, columns of every tile, against the oracle."""
    M, N, K = 2048, 4864, 2048
    Wh = wq_inputs.weight_f16(31, 0, N, K)
    x = wq_inputs.activations_bf16(31, 1, M, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).float().cpu().numpy()
    assert m.wq_last_device_error() == m.WQ_OK
    rng = np.random.default_rng(10)
    cols = np.unique(np.concatenate([np.arange(0, N, 256), np.arange(255, N, 256), rng.integers(0, N, 40)]))
    rows = np.unique(np.concatenate([[0, 255, 1792, M - 1], rng.integers(0, 256, 6), rng.integers(1792, M, 10)]))
    oc, os_, oz = oracle_quantize(Wh[cols], bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x[torch.from_numpy(rows)]), oc, os_, oz, len(cols), K, bits, group)
    assert_y_close(y[np.ix_(rows, cols)], y_ref, bound, f"152 tiles bits={bits} g={group}")


def test_tc_two_launches_keep_stream_order():
    """With 152 tiles the GEMM runs as a launch of 148 whole tiles and a
    dependent launch of the 4 left over, which may start before the first
    ends.  Work queued right behind the GEMM on its stream (here a copy of y)
    must still see every tile of both launches."""
    M, N, K, bits, group = 2048, 4864, 2048, 4, 128
    m = wq()
    Wh = wq_inputs.weight_f16(32, 0, N, K)
    x = wq_inputs.activations_bf16(32, 1, M, K).cuda()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    ref = m.wq_gemm(x, codes, s, z, bits, group, N, K)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    for _ in range(3):
        y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            m.wq_gemm(x, codes, s, z, bits, group, N, K, y=y, stream=side)
            snap = y.clone()
        side.synchronize()
        assert m.wq_last_device_error() == m.WQ_OK
        assert torch.equal(snap, ref)
        assert torch.equal(y, ref)
