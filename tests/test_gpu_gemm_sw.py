"""Batches of 17..255 rows on the tensor cores with the weight rows on the
MMA's M side (gemm_sw) vs the oracle: y within the stated tolerance on every
token tile (32, 64, 128, 256 columns), ragged N, per-row grids and groups of
64..384, split-K clusters, sampled rows of full-size layers, and one-hot
exactness (y = bf16(w') for a one-hot x)."""
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
@pytest.mark.parametrize("M", [17, 32, 33, 64, 65, 128, 129, 200, 255])
def test_sw_token_tiles(bits, M):
    N, K, group = 300, 1152, 128            # ragged N (3 tiles), 9 code stages
    Wh = wq_inputs.weight_f16(80, bits, N, K, dist="t4")
    x = wq_inputs.activations_bf16(80, M, M, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, f"bits={bits} M={M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("N,K,group", [(256, 2048, 0), (130, 1280, 256), (200, 768, 384), (64, 4096, 64),
                                       (128, 11008, 128), (96, 13824, 0)])
def test_sw_groups_and_splits(bits, N, K, group):
    """Per-row grids (scale in the epilogue), groups of 64..384, and few
    128-row tiles over a long K (split-K clusters of up to 8 CTAs)."""
    Wh = wq_inputs.weight_f16(81, bits, N, K, dist="t4")
    for M in (24, 100):
        x = wq_inputs.activations_bf16(81, M, M, K)
        y, yr, b = _run(Wh, x, bits, group)
        assert_y_close(y, yr, b, f"bits={bits} N={N} K={K} g={group} M={M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", [128, 0])
def test_sw_one_hot_exact(bits, group):
    """Token m is one-hot at column k_m: the MMA meets one bf16 w' (grouped
    grids) or one exact q - z times the fp32 row scale (per-row grids), so y
    must equal bf16(c w') exactly; every other token row is zero."""
    N, K = 256, 1024
    Wh = wq_inputs.weight_f16(82, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    w_ref = torch.from_numpy(oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group))
    for M in (20, 64, 150):
        x = torch.zeros(M, K, dtype=torch.bfloat16)
        ks = [(7 * i + 3) % K for i in range(0, M, 3)]
        for i, k in zip(range(0, M, 3), ks):
            x[i, k] = 2.0 if i % 2 else -1.0
        y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
        for i, k in zip(range(0, M, 3), ks):
            ref = ((2.0 if i % 2 else -1.0) * w_ref[:, k]).to(torch.bfloat16)
            assert torch.equal(y[i], ref), (M, i, k)
        others = [i for i in range(M) if i % 3]
        assert torch.equal(y[others], torch.zeros(len(others), N, dtype=torch.bfloat16))


@pytest.mark.parametrize("cfg,linear,M", [
    ("llama7b_stack32_4b_g128", 0, 64), ("llama7b_stack32_4b_g128", 4, 64), ("llama7b_stack32_4b_g128", 6, 64),
    ("llama7b_layer_3b_g128", 0, 33), ("llama7b_layer_3b_g128", 3, 17),
    ("llama13b_prefill_4b_g128", 0, 128), ("llama13b_prefill_4b_g128", 1, 200),
    ("opt175b_fc_2b_rowwise", 1, 48)])
def test_sw_full_size_sampled(cfg, linear, M):
    w = wq_inputs.WORKLOADS[cfg]
    name, N, K = w["linears"][linear]
    bits, group = w["bits"], w["group"]
    Wh = cached_weight(0, linear, N, K, w["dist"])
    x = wq_inputs.activations_bf16(0, 600 + linear, M, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).float().cpu().numpy()
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(linear).integers(0, N, 126)]))
    oc, os_, oz = oracle_quantize(Wh[cols], bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, len(cols), K, bits, group)
    assert_y_close(y[:, cols], y_ref, bound, f"{cfg}/{name} M={M}")


def test_sw_no_write_beyond_y_and_zero_x():
    N, K, bits, group, M = 200, 512, 4, 128, 40
    Wh = wq_inputs.weight_f16(83, 0, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    x = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    buf = torch.full((M * N + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    y = buf[32:32 + M * N].view(M, N)
    m.wq_gemm(x, codes, s, z, bits, group, N, K, y=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    assert torch.all(buf[:32] == 7.0) and torch.all(buf[32 + M * N:] == 7.0)
