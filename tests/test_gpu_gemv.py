"""Decode GEMV (M <= 16) vs the oracle: y within the stated tolerance."""
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
    """Quantise on the GPU, multiply on the GPU; oracle from the same host bytes."""
    N, K = Wh.shape
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K)
    torch.cuda.synchronize()
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, N, K, bits, group)
    return y.float().cpu().numpy(), y_ref, bound


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 13, 16])
def test_gemv_small(bits, M):
    N, K, group = 70, 640, 128          # ragged N (3 CTAs), 20 blocks over 8 warps
    Wh = wq_inputs.weight_f16(4, bits, N, K)
    x = wq_inputs.activations_bf16(4, M, M, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, f"bits={bits} M={M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group,K", [(32, 96), (64, 192), (0, 32), (0, 4160), (96, 288)])
def test_gemv_groups_and_edges(bits, group, K):
    N = 33
    Wh = wq_inputs.weight_f16(5, bits, N, K, dist="t4")
    for M in (1, 7):
        x = wq_inputs.activations_bf16(5, M, M, K)
        y, yr, b = _run(Wh, x, bits, group)
        assert_y_close(y, yr, b, f"bits={bits} group={group} K={K} M={M}")


@pytest.mark.parametrize("bits", BITS)
def test_gemv_one_hot_exact(bits):
    """A one-hot x selects one column of W': y must equal bf16(w') exactly."""
    N, K, group = 64, 256, 64
    Wh = wq_inputs.weight_f16(6, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    wq_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
    for k in (0, 5, 31, 32, 100, 255):
        x = torch.zeros(3, K, dtype=torch.bfloat16)
        x[0, k] = 1.0
        x[2, k] = -2.0
        y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
        ref = torch.from_numpy(wq_ref[:, k]).to(torch.bfloat16)
        assert torch.equal(y[0], ref)
        assert torch.equal(y[1], torch.zeros(N, dtype=torch.bfloat16))
        assert torch.equal(y[2], (-2.0 * torch.from_numpy(wq_ref[:, k])).to(torch.bfloat16))


def test_gemv_zero_x_and_no_overwrite_beyond_y():
    N, K, bits, group = 40, 128, 4, 32
    Wh = wq_inputs.weight_f16(7, 0, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    x = torch.zeros(2, K, dtype=torch.bfloat16, device="cuda")
    buf = torch.full((2 * N + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    y = buf[32:32 + 2 * N].view(2, N)
    m.wq_gemm(x, codes, s, z, bits, group, N, K, y=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    assert torch.all(buf[:32] == 7.0) and torch.all(buf[32 + 2 * N:] == 7.0)


@pytest.mark.parametrize("cfg,linear,M", [
    ("linear4096_4b_g128", 0, 1),
    ("llama7b_layer_3b_g128", 0, 1), ("llama7b_layer_3b_g128", 1, 4),
    ("llama7b_layer_3b_g128", 2, 16), ("llama7b_layer_3b_g128", 3, 1),
    ("opt175b_fc_2b_rowwise", 0, 1), ("opt175b_fc_2b_rowwise", 1, 1),
    ("opt175b_fc_8b_rowwise", 0, 1), ("opt175b_fc_8b_rowwise", 1, 1),
    ("llama7b_stack32_4b_g128", 6, 16)])
def test_gemv_full_size_sampled(cfg, linear, M):
    w = wq_inputs.WORKLOADS[cfg]
    name, N, K = w["linears"][linear]
    bits, group = w["bits"], w["group"]
    Wh = cached_weight(0, linear, N, K, w["dist"])
    x = wq_inputs.activations_bf16(0, 100 + linear, M, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).float().cpu().numpy()
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(7).integers(0, N, 126)]))
    oc, os_, oz = oracle_quantize(Wh[cols], bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, len(cols), K, bits, group)
    assert_y_close(y[:, cols], y_ref, bound, f"{cfg}/{name} M={M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group,K", [(32, 8192), (32, 12416), (64, 16512)])
def test_gemv_m1_long_k(bits, group, K):
    """M = 1 over K ranges whose scale groups outnumber one shared table:
    the table is reloaded between stages; the last stage is ragged."""
    N = 70
    Wh = wq_inputs.weight_f16(8, bits, N, K)
    x = wq_inputs.activations_bf16(8, 1, 1, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, f"bits={bits} g={group} K={K}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("offset", [1, 4, 8])
def test_gemv_m1_offset_x(bits, offset):
    """x starting 2, 8 or 16 bytes into a buffer: the C ABI takes 16-byte
    aligned pointers only, so the first two are refused with status 5 and the
    third is served."""
    N, K, group = 70, 1280, 128
    Wh = wq_inputs.weight_f16(9, bits, N, K)
    x = wq_inputs.activations_bf16(9, 1, 1, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    buf = torch.zeros(K + 16, dtype=torch.bfloat16, device="cuda")
    buf[offset:offset + K] = x[0].cuda()
    xv = buf[offset:offset + K].view(1, K)
    if offset * 2 % 16:
        with pytest.raises(m.WQError) as e:
            m.wq_gemm(xv, codes, s, z, bits, group, N, K)
        assert e.value.status == 5
        return
    y = m.wq_gemm(xv, codes, s, z, bits, group, N, K)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, N, K, bits, group)
    assert_y_close(y.float().cpu().numpy(), y_ref, bound, f"bits={bits} offset={offset}")


@pytest.mark.parametrize("bits", BITS)
def test_gemv_m1_one_hot_exact(bits):
    """M = 1 with a one-hot x: y must equal bf16(w') of that column exactly,
    including columns in the ragged last stage."""
    N, K, group = 64, 1152, 64
    Wh = wq_inputs.weight_f16(10, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    wq_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
    for k in (0, 31, 1023, 1024, 1151):
        x = torch.zeros(1, K, dtype=torch.bfloat16)
        x[0, k] = 1.0
        y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
        assert torch.equal(y[0], torch.from_numpy(wq_ref[:, k]).to(torch.bfloat16))


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("N,K,group", [(70, 1152, 128), (70, 1152, 384), (33, 2048, 0), (100, 5120, 256),
                                       (40, 128, 128)])
def test_gemv_m1_tma_groups(bits, N, K, group):
    """M = 1 with K a multiple of 128 (TMA-staged codes): ragged N, a 128-code
    last stage at K = 1152, groups of 128, 256 and 384 and a per-row grid."""
    Wh = wq_inputs.weight_f16(11, bits, N, K, dist="t4")
    x = wq_inputs.activations_bf16(11, 1, 1, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, f"bits={bits} N={N} K={K} g={group}")


@pytest.mark.parametrize("bits", BITS)
def test_gemv_m1_one_hot_exact_g128(bits):
    """M = 1, g = 128, one nonzero x: a single exact product per row, so
    y = bf16(-3 w') exactly."""
    N, K, group = 64, 1152, 128
    Wh = wq_inputs.weight_f16(12, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    wq_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
    for k in (0, 5, 31, 127, 128, 1023, 1024, 1151):
        x = torch.zeros(1, K, dtype=torch.bfloat16)
        x[0, k] = -3.0
        y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
        assert torch.equal(y[0], (-3.0 * torch.from_numpy(wq_ref[:, k])).to(torch.bfloat16)), k


def test_gemv_m1_table_windows_g128():
    """N = 14240, K = 16512, g = 128: one CTA's K range spans 129 groups, more
    than its scale table holds, so the table is reloaded between stages;
    checked on sampled rows."""
    N, K, bits, group = 14240, 16512, 2, 128
    Wh = wq_inputs.weight_f16(13, bits, N, K)
    x = wq_inputs.activations_bf16(13, 1, 1, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).float().cpu().numpy()
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(9).integers(0, N, 126)]))
    oc, os_, oz = oracle_quantize(Wh[cols], bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, len(cols), K, bits, group)
    assert_y_close(y[:, cols], y_ref, bound, "table windows")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [2, 3, 6, 8])
@pytest.mark.parametrize("N,K,group", [(70, 1152, 128), (33, 2048, 0), (100, 1280, 256)])
def test_gemv_small_batch_quads(bits, M, N, K, group):
    """2..8 tokens with K and the group length in whole 128-code quads (the
    warp-level MMA GEMV): ragged N, a one-quad last stage, per-row grids."""
    Wh = wq_inputs.weight_f16(14, bits, N, K, dist="t4")
    x = wq_inputs.activations_bf16(14, M, M, K)
    y, yr, b = _run(Wh, x, bits, group)
    assert_y_close(y, yr, b, f"bits={bits} M={M} N={N} K={K} g={group}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [2, 5, 8])
def test_gemv_small_batch_one_hot_exact_g128(bits, M):
    """2..8 tokens, g = 128: token m is one-hot at column k_m (one exact
    product per output), the last token is all zero."""
    N, K, group = 64, 1152, 128
    Wh = wq_inputs.weight_f16(15, bits, N, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    wq_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
    ks = [0, 31, 127, 128, 1023, 1024, 1151, 600][:M - 1]
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    for i, k in enumerate(ks):
        x[i, k] = 2.0 if i % 2 else -1.0
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).cpu()
    for i, k in enumerate(ks):
        ref = ((2.0 if i % 2 else -1.0) * torch.from_numpy(wq_ref[:, k])).to(torch.bfloat16)
        assert torch.equal(y[i], ref), (i, k)
    assert torch.equal(y[M - 1], torch.zeros(N, dtype=torch.bfloat16))


def _sampled_case(seed, N, K, bits, group, M, what):
    """Full GPU quantise + GEMV; the oracle on 128 sampled output rows."""
    Wh = wq_inputs.weight_f16(seed, bits, N, K)
    x = wq_inputs.activations_bf16(seed, M, M, K)
    m = wq()
    codes, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    y = m.wq_gemm(x.cuda(), codes, s, z, bits, group, N, K).float().cpu().numpy()
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(seed).integers(0, N, 126)]))
    oc, os_, oz = oracle_quantize(Wh[cols], bits, group)
    y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, len(cols), K, bits, group)
    assert_y_close(y[:, cols], y_ref, bound, what)


@pytest.mark.parametrize("bits", (3, 4))
@pytest.mark.parametrize("M", [2, 4, 8])
def test_gemv_small_batch_split_k_cluster(bits, M):
    """2..8 tokens, N = 4096, K = 11008, g = 128 (the 7B down projection):
    the warp-MMA GEMV splits K over a 2-CTA cluster and adds the partial sums
    through distributed shared memory."""
    _sampled_case(16, 4096, 11008, bits, 128, M, f"split-K bits={bits} M={M}")


def test_gemv_small_batch_table_windows_g128():
    """4 tokens, N = 14240, K = 16512, g = 128: one CTA's K range spans 129
    scale groups, more than its shared table holds, so the warp-MMA GEMV
    reloads the table between stages."""
    _sampled_case(17, 14240, 16512, 2, 128, 4, "warp-MMA table windows")
