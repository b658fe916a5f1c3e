"""wq_gemm_grouped_noalloc: the grouped decode GEMV on the library's built-in
workspace, for callers that cannot allocate device memory when they call (a
runtime that owns all GPU memory through its own pool, code running during
CUDA graph capture, a decode loop where an allocation could stall or fail).

Called through the C ABI twice in a row on the same linears (the second call
reuses the built-in array as the first call left it), each result is compared
with wq_gemm_grouped's (the entry point that takes a caller workspace) within
the tolerance the parity tests use.  A call that needs more workspace than the
built-in 8 MiB is refused before anything runs.  This file runs last so that a
failure here leaves every other test already run; it needs nothing from them.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from gpu_util import ABS_TOL, OUT_ROUND, REL_TOL, oracle_quantize, to_dev_f16, wq

pytestmark = pytest.mark.gpu


def _linears(m, bits, shapes, M, seed):
    items, refs = [], []
    for i, (N, K, group) in enumerate(shapes):
        Wh = wq_inputs.weight_f16(seed, i, N, K)
        c, s, z = m.wq_quantize_rtn(to_dev_f16(Wh), bits, group)
        x = wq_inputs.activations_bf16(seed, 10 + i, M, K)
        items.append((x.cuda(), c, s, z, N, K, group))
        refs.append((Wh, x))
    return items, refs


def _bound(Wh, x, bits, group):
    N, K = Wh.shape
    oc, os_, oz = oracle_quantize(Wh, bits, group)
    _, b = oracle.gemm(wq_inputs.bf16_bits(x), oc, os_, oz, N, K, bits, group)
    return b


def _call_noalloc(m, items, bits, ys):
    arr = (m.Linear * len(items))()
    for i, ((x, c, s, z, N, K, g), y) in enumerate(zip(items, ys)):
        arr[i] = m.Linear(x.data_ptr(), c.data_ptr(), s.data_ptr(), z.data_ptr(), y.data_ptr(), N, K, g)
    return m.lib.wq_gemm_grouped_noalloc(arr, len(items), items[0][0].shape[0], bits,
                                         torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("bits,M", [(4, 1), (3, 4), (4, 16)])
def test_noalloc_matches_workspace_entry_point_twice(bits, M):
    m = wq()
    shapes = [(4096, 4096, 128), (1000, 1152, 128), (300, 2048, 0)]
    items, refs = _linears(m, bits, shapes, M, seed=70 + M)
    ref_ys = m.wq_gemm_grouped(items, bits)
    torch.cuda.synchronize()
    bounds = [_bound(Wh, x, bits, g) for (Wh, x), (_, _, g) in zip(refs, shapes)]
    for _ in range(2):
        ys = [torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda") for (N, _, _) in shapes]
        assert _call_noalloc(m, items, bits, ys) == m.WQ_OK
        torch.cuda.synchronize()
        for y, r, b in zip(ys, ref_ys, bounds):
            a, e = y.float().cpu().numpy().astype(np.float64), r.float().cpu().numpy().astype(np.float64)
            assert np.all(np.abs(a - e) <= REL_TOL * b + OUT_ROUND * np.abs(e) + ABS_TOL)
    assert m.wq_last_device_error() == m.WQ_OK


def test_noalloc_refuses_more_than_its_workspace():
    m = wq()
    bits, M = 4, 16
    # 48 linears of K = 11008 at 16 tokens need about 17 MiB of workspace
    W = torch.zeros(64, 11008, dtype=torch.float16, device="cuda")
    c, s, z = m.wq_quantize_rtn(W, bits, 128)
    x = torch.zeros(M, 11008, dtype=torch.bfloat16, device="cuda")
    items = [(x, c, s, z, 64, 11008, 128) for _ in range(48)]
    assert m.grouped_workspace_size(items, bits) > 8 << 20
    ys = [torch.full((M, 64), 7.0, dtype=torch.bfloat16, device="cuda") for _ in items]
    assert _call_noalloc(m, items, bits, ys) == m.WQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert all(bool(torch.all(y == 7.0)) for y in ys)
