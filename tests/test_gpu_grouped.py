"""Grouped calls (wq_gemm_grouped) vs the oracle: every y of a list of linears
within the stated tolerance, one-hot exactness, determinism, stream-K splits of
a tile between CTAs, several launches sharing one workspace, nothing written
outside y; at 1..16 rows the persistent decode GEMV, at 17..255 rows the
swap-AB tensor-core GEMM in grouped launches."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from gpu_util import assert_y_close, cached_weight, oracle_quantize, to_dev_f16, wq

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)
# (N, K, group): ragged N, a ragged last stage (K = 1152, 1280), per-row grids,
# groups of 128/256/384, and one linear the persistent kernel does not take
# (K = 96, group 32), which runs as wq_gemm would.
SHAPES = [(70, 1152, 128), (33, 2048, 0), (100, 1280, 256), (64, 4096, 128), (45, 1152, 384),
          (40, 96, 32), (300, 640, 128)]


def _quantized(seed, shapes, bits, dist="normal"):
    m = wq()
    out = []
    for i, (N, K, group) in enumerate(shapes):
        Wh = wq_inputs.weight_f16(seed, 10 * bits + i, N, K, dist=dist)
        c, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
        out.append((Wh, c, s, z, N, K, group))
    return out


def _check_all(qs, xs, ys, bits, what, rows=None):
    for i, ((Wh, c, s, z, N, K, group), x, y) in enumerate(zip(qs, xs, ys)):
        yv = y.float().cpu().numpy()
        sel = np.arange(N) if rows is None else rows[i]
        oc, os_, oz = oracle_quantize(Wh[sel], bits, group)
        y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, len(sel), K, bits, group)
        assert_y_close(yv[:, sel], y_ref, bound, f"{what} linear {i} (N={N} K={K} g={group})")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 13, 16])
def test_grouped_small(bits, M):
    qs = _quantized(20, SHAPES, bits, dist="t4")
    xs = [wq_inputs.activations_bf16(20, 100 + i, M, K) for i, (_, K, _) in enumerate(SHAPES)]
    m = wq()
    items = [(x.cuda(), c, s, z, N, K, g) for x, (_, c, s, z, N, K, g) in zip(xs, qs)]
    ys = m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    _check_all(qs, xs, ys, bits, f"bits={bits} M={M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [1, 6, 16])
def test_grouped_one_hot_exact(bits, M):
    """Token m is one-hot at column k_m (one exact product per output), the
    last token all zero: y must equal bf16(c w') exactly."""
    shapes = [(64, 1152, 128), (40, 2048, 0)]
    qs = _quantized(21, shapes, bits)
    m = wq()
    ks = [0, 31, 127, 128, 1023, 1024, 1151, 600, 5, 77, 900, 1100, 256, 512, 1000, 64]
    items, xs, refs = [], [], []
    for (Wh, c, s, z, N, K, group) in qs:
        oc, os_, oz = oracle_quantize(Wh, bits, group)
        w_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
        x = torch.zeros(M, K, dtype=torch.bfloat16)
        r = []
        for i in range(M - 1 if M > 1 else 1):
            k = ks[i] % K
            v = 2.0 if i % 2 else -1.0
            x[i, k] = v
            r.append((i, (v * torch.from_numpy(w_ref[:, k])).to(torch.bfloat16)))
        xs.append(x)
        refs.append(r)
        items.append((x.cuda(), c, s, z, N, K, group))
    ys = [y.cpu() for y in m.wq_gemm_grouped(items, bits)]
    for y, r, (_, _, _, _, N, _, _) in zip(ys, refs, qs):
        for i, ref in r:
            assert torch.equal(y[i], ref), i
        if M > 1:
            assert torch.equal(y[M - 1], torch.zeros(N, dtype=torch.bfloat16))


@pytest.mark.parametrize("M", [1, 4, 16])
def test_grouped_deterministic_and_workspace_reset(M):
    """Two calls give identical bits; every tile counter is back at zero."""
    bits = 4
    shapes = [(4096, 4096, 128), (11008, 4096, 128), (4096, 11008, 128)]
    qs = _quantized(22, shapes, bits)
    m = wq()
    xs = [wq_inputs.activations_bf16(22, 200 + i, M, K).cuda() for i, (_, K, _) in enumerate(shapes)]
    items = [(x, c, s, z, N, K, g) for x, (_, c, s, z, N, K, g) in zip(xs, qs)]
    ws = m.grouped_workspace(items, bits)
    y1 = [y.clone() for y in m.wq_gemm_grouped(items, bits, workspace=ws)]
    y2 = m.wq_gemm_grouped(items, bits, workspace=ws)
    torch.cuda.synchronize()
    for a, b in zip(y1, y2):
        assert torch.equal(a, b)
    assert int(ws[:4096].count_nonzero()) == 0
    rows = [np.unique(np.concatenate([[0, N - 1], np.random.default_rng(i).integers(0, N, 62)]))
            for i, (N, _, _) in enumerate(shapes)]
    _check_all(qs, [x.cpu() for x in xs], y1, bits, f"M={M}", rows=rows)


def test_grouped_single_small_linear_split_tiles():
    """One 4096 x 4096 linear (128 row tiles over every CTA): nearly every
    tile is cut between CTAs and finished through the workspace."""
    bits, N, K, group = 4, 4096, 4096, 128
    Wh = cached_weight(0, 0, N, K, "normal")
    m = wq()
    c, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
    for M in (1, 3, 16):
        x = wq_inputs.activations_bf16(23, M, M, K)
        (y,) = m.wq_gemm_grouped([(x.cuda(), c, s, z, N, K, group)], bits)
        rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(M).integers(0, N, 254)]))
        _check_all([(Wh, c, s, z, N, K, group)], [x], [y], bits, f"single M={M}", rows=[rows])


def test_grouped_many_linears_share_workspace():
    """130 linears: two persistent launches (at most 128 linears each) reuse
    the workspace's counters and partial-sum slots in stream order."""
    bits = 3
    shapes = [(32 + (i % 5) * 17, 128 * (1 + i % 9), 128 if i % 3 else 0) for i in range(130)]
    qs = _quantized(24, shapes, bits)
    m = wq()
    xs = [wq_inputs.activations_bf16(24, 300 + i, 2, K) for i, (_, K, _) in enumerate(shapes)]
    items = [(x.cuda(), c, s, z, N, K, g) for x, (_, c, s, z, N, K, g) in zip(xs, qs)]
    ys = m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    _check_all(qs, xs, ys, bits, "130 linears")


@pytest.mark.parametrize("cfg,M", [("llama7b_layer_3b_g128", 1), ("llama7b_layer_3b_g128", 4),
                                   ("llama7b_layer_3b_g128", 16), ("opt175b_fc_2b_rowwise", 1),
                                   ("opt175b_fc_8b_rowwise", 1), ("llama7b_stack32_4b_g128", 1),
                                   ("llama7b_stack32_4b_g128", 16)])
def test_grouped_full_size_sampled(cfg, M):
    """The workloads' linears in one grouped call (the stack: its first layer),
    each checked on 128 sampled output rows."""
    w = wq_inputs.WORKLOADS[cfg]
    lins = w["linears"][:7]
    bits, group = w["bits"], w["group"]
    m = wq()
    qs, items, xs, rows = [], [], [], []
    for i, (name, N, K) in enumerate(lins):
        Wh = cached_weight(0, i, N, K, w["dist"])
        c, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
        x = wq_inputs.activations_bf16(0, 400 + i, M, K)
        qs.append((Wh, c, s, z, N, K, group))
        xs.append(x)
        items.append((x.cuda(), c, s, z, N, K, group))
        rows.append(np.unique(np.concatenate([[0, N - 1], np.random.default_rng(i).integers(0, N, 126)])))
    ys = m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    _check_all(qs, xs, ys, bits, f"{cfg} M={M}", rows=rows)


def test_grouped_no_write_outside_y_and_small_workspace_refused():
    bits, N, K, group = 4, 96, 1024, 128
    (Wh, c, s, z, _, _, _), = _quantized(25, [(N, K, group)], bits)
    m = wq()
    x = wq_inputs.activations_bf16(25, 0, 2, K).cuda()
    buf = torch.full((2 * N + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    y = buf[32:32 + 2 * N].view(2, N)
    items = [(x, c, s, z, N, K, group, y)]
    need = m.grouped_workspace_size(items, bits)
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.WQError) as e:
        m.wq_gemm_grouped(items, bits, workspace=small)
    assert e.value.status == m.WQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(buf == 7.0)
    m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    assert torch.all(buf[:32] == 7.0) and torch.all(buf[32 + 2 * N:] == 7.0)
    _check_all([(Wh, c, s, z, N, K, group)], [x.cpu()], [y], bits, "canaries")


# 17..255 rows: the swap-AB tensor-core GEMM in grouped launches (one CTA per
# 128-row tile over all of K); the K = 96 linear still runs as wq_gemm would.
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [17, 33, 64, 100, 255])
def test_grouped_swap_ab(bits, M):
    qs = _quantized(26, SHAPES, bits, dist="t4")
    xs = [wq_inputs.activations_bf16(26, 500 + i, M, K) for i, (_, K, _) in enumerate(SHAPES)]
    m = wq()
    items = [(x.cuda(), c, s, z, N, K, g) for x, (_, c, s, z, N, K, g) in zip(xs, qs)]
    ys = m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    _check_all(qs, xs, ys, bits, f"swap-AB grouped bits={bits} M={M}")


@pytest.mark.parametrize("bits", (2, 4, 8))
def test_grouped_swap_ab_one_hot_exact(bits):
    """One-hot tokens (the last all zero) through the grouped swap-AB launch:
    y must equal bf16(c w') exactly, per-row and grouped grids."""
    shapes = [(200, 1152, 128), (130, 2048, 0)]
    qs = _quantized(27, shapes, bits)
    M = 40
    m = wq()
    items, refs = [], []
    for (Wh, c, s, z, N, K, group) in qs:
        oc, os_, oz = oracle_quantize(Wh, bits, group)
        w_ref = oracle.dequant(oracle.unpack(oc, K, bits), os_, oz, group)
        x = torch.zeros(M, K, dtype=torch.bfloat16)
        r = []
        for i in range(M - 1):
            k = (37 * i + 5) % K
            v = 2.0 if i % 2 else -1.0
            x[i, k] = v
            r.append((i, (v * torch.from_numpy(w_ref[:, k])).to(torch.bfloat16)))
        refs.append(r)
        items.append((x.cuda(), c, s, z, N, K, group))
    ys = [y.cpu() for y in m.wq_gemm_grouped(items, bits)]
    for y, r in zip(ys, refs):
        for i, want in r:
            assert torch.equal(y[i], want), f"token {i}"
        assert torch.all(y[M - 1] == 0)


def test_grouped_swap_ab_many_linears_and_noalloc():
    """150 linears at 48 rows: three grouped launches (at most 64 linears
    each); the no-alloc entry gives the same bits (no workspace is used)."""
    bits = 4
    shapes = [(64 + (i % 7) * 40, 128 * (1 + i % 6), 128 if i % 4 else 0) for i in range(150)]
    qs = _quantized(28, shapes, bits)
    m = wq()
    M = 48
    xs = [wq_inputs.activations_bf16(28, 600 + i, M, K) for i, (_, K, _) in enumerate(shapes)]
    items = [(x.cuda(), c, s, z, N, K, g) for x, (_, c, s, z, N, K, g) in zip(xs, qs)]
    ys = m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    _check_all(qs, xs, ys, bits, "150 linears at 48 rows")
    items2 = [it + (torch.empty(M, it[4], dtype=torch.bfloat16, device="cuda"),) for it in items]
    ys2 = m.wq_gemm_grouped_noalloc(items2, bits)
    torch.cuda.synchronize()
    for a, b in zip(ys, ys2):
        assert torch.equal(a, b)
