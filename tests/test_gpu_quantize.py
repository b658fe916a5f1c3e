"""GPU quantiser vs the oracle: codes, scales and zeros bit-exact."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from gpu_util import cached_weight, gpu_quantize, oracle_quantize, wq

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)


def _assert_same(Wh, bits, group):
    gc, gs, gz = gpu_quantize(Wh, bits, group)
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    assert np.array_equal(gs, os_), "scales differ"
    assert np.array_equal(gz, oz), "zeros differ"
    assert np.array_equal(gc, oc), "codes differ"


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", [32, 64, 128, 0, 96])
def test_quantize_small_matrices(bits, group):
    # K spans several blocks with a ragged group count; N ragged.
    K = 384 if group != 96 else 480
    for dist in ("normal", "t4"):
        Wh = wq_inputs.weight_f16(1, bits, 37, K, dist=dist)
        _assert_same(Wh, bits, group)


@pytest.mark.parametrize("bits", BITS)
def test_quantize_long_rows(bits):
    # per-row grids longer than 32 blocks take the CTA-per-row kernel
    Wh = wq_inputs.weight_f16(2, bits, 9, 11008, dist="t4")
    _assert_same(Wh, bits, 0)
    _assert_same(Wh, bits, 5504 if 5504 % 32 == 0 else 0)


@pytest.mark.parametrize("bits", BITS)
def test_quantize_edge_groups(bits):
    rng = np.random.default_rng(3)
    rows = [np.zeros(64), np.full(64, 1e-8), -np.abs(rng.standard_normal(64)),
            np.abs(rng.standard_normal(64)) * 100, rng.standard_normal(64) * 1e-6,
            rng.integers(-8, 8, 64) * 2.0 ** -5, np.full(64, 65504.0),
            np.concatenate([[-65504.0, 65504.0], rng.standard_normal(62)]),
            np.where(rng.random(64) < 0.5, -0.0, 0.0)]
    Wh = np.array(rows).astype(np.float16)
    for group in (32, 64):
        _assert_same(Wh, bits, group)


def test_quantize_exhaustive_fp16_sweep():
    """Every finite fp16 value, quantised inside groups whose min/max pin a
    range of scales (normal and subnormal), bit-exact with the oracle."""
    from exact import ALL_FINITE_F16
    vals = ALL_FINITE_F16.view(np.float16)
    rows = []
    for lo, hi in [(-1.0, 1.0), (-65504.0, 65504.0), (-6e-5, 3e-5), (-1e-7, 2e-7),
                   (-0.07, 0.0), (0.0, 300.0), (-2.0 ** -14, 2.0 ** -14)]:
        inside = vals[(vals.astype(np.float64) >= lo) & (vals.astype(np.float64) <= hi)]
        per = 30
        n = (inside.size + per - 1) // per
        pad = np.resize(inside, n * per).reshape(n, per)
        blk = np.concatenate([np.full((n, 1), lo), np.full((n, 1), hi), pad.astype(np.float64)], 1)
        rows.append(blk)
    Wh = np.concatenate(rows).astype(np.float16)
    for bits in BITS:
        _assert_same(Wh, bits, 32)


@pytest.mark.parametrize("cfg,linear", [
    ("linear4096_4b_g128", 0), ("llama7b_layer_3b_g128", 0), ("llama7b_layer_3b_g128", 3),
    ("opt175b_fc_2b_rowwise", 1), ("opt175b_fc_8b_rowwise", 0), ("llama13b_prefill_4b_g128", 1)])
def test_quantize_full_size_sampled_rows(cfg, linear):
    w = wq_inputs.WORKLOADS[cfg]
    name, N, K = w["linears"][linear]
    Wh = cached_weight(0, linear, N, K, w["dist"])
    gc, gs, gz = gpu_quantize(Wh, w["bits"], w["group"])
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(linear).integers(0, N, 62)]))
    oc, os_, oz = oracle_quantize(Wh[rows], w["bits"], w["group"])
    assert np.array_equal(gs[rows], os_) and np.array_equal(gz[rows], oz)
    assert np.array_equal(gc[rows], oc)
