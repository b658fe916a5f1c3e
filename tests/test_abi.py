"""The C-ABI library loads on a host without a GPU, exports every function
include/wq.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wq():
    import quantized_gemm_wq_b200 as wq
    return wq


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "wq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_function(wq):
    names = _declared_functions()
    assert set(names) == set(wq.EXPORTED)
    for n in names:
        assert hasattr(wq.lib, n), n


def test_layout_helpers(wq):
    assert wq.wq_codes_words(4096, 4096, 4) == 4096 * 4096 * 4 // 32
    assert wq.wq_codes_words(3, 96, 3) == 3 * 9
    assert wq.wq_codes_words(3, 40, 3) == 0
    assert wq.wq_codes_words(3, 64, 5) == 0
    assert wq.wq_params_count(4096, 4096, 128) == 4096 * 32
    assert wq.wq_params_count(5, 4096, 0) == 5
    assert wq.wq_params_count(5, 4096, 4096) == 5
    assert wq.wq_params_count(5, 4096, 48) == 0


def test_status_strings(wq):
    for s in range(10):
        assert len(wq.wq_status_string(s)) >= 2
    assert "unknown" in wq.wq_status_string(99)


def test_rejects_before_device(wq):
    L = wq.lib
    P = 1 << 20          # a non-null, 16-byte aligned fake address: never dereferenced
    q = L.wq_quantize_rtn
    assert q(None, 4, 64, 4, 32, P, P, P, None) == wq.WQ_ERR_NULL
    assert q(P, 4, 64, 5, 32, P, P, P, None) == wq.WQ_ERR_BITS
    assert q(P, 4, 63, 4, 0, P, P, P, None) == wq.WQ_ERR_SHAPE
    assert q(P, 0, 64, 4, 0, P, P, P, None) == wq.WQ_ERR_SHAPE
    assert q(P, 4, 64, 4, 48, P, P, P, None) == wq.WQ_ERR_GROUP
    assert q(P, 4, 64, 4, 16, P, P, P, None) == wq.WQ_ERR_GROUP
    assert q(P + 8, 4, 64, 4, 32, P, P, P, None) == wq.WQ_ERR_ALIGN
    g = L.wq_gemm
    assert g(P, 1, 4, 64, P, P, P, 4, 32, None, None) == wq.WQ_ERR_NULL
    assert g(P, 0, 4, 64, P, P, P, 4, 32, P, None) == wq.WQ_ERR_SHAPE
    assert g(P, 1, 4, 64, P, P, P, 7, 32, P, None) == wq.WQ_ERR_BITS
    assert g(P, 1, 4, 64, P, P, P, 4, 96, P, None) == wq.WQ_ERR_GROUP
    assert g(P, 1, 4, 64, P, P, P + 4, 4, 32, P, None) == wq.WQ_ERR_ALIGN


def test_binding_checks_tensors_before_the_library(wq):
    """The Python binding refuses host tensors, wrong dtypes and mismatched
    shapes itself, before any pointer reaches the C ABI."""
    import torch
    c = torch.zeros(4, 8, dtype=torch.int32)
    s = torch.zeros(4, 2, dtype=torch.float16)
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        wq.wq_gemm(x, c, s, s, 4, 32, 4, 64)                      # host tensor
    with pytest.raises(ValueError):
        wq.wq_gemm(x.float(), c, s, s, 4, 32, 4, 64)              # not bf16
    with pytest.raises(ValueError):
        wq.wq_gemm(torch.zeros(64, dtype=torch.bfloat16), c, s, s, 4, 32, 4, 64)   # not 2-D
    with pytest.raises(ValueError):
        wq.wq_quantize_rtn(torch.zeros(4, 64, dtype=torch.float32), 4, 32)          # not fp16
    with pytest.raises(ValueError):
        wq.wq_quantize_rtn(torch.zeros(4, 64, dtype=torch.float16).t(), 4, 32)      # not contiguous


def test_grouped_rejects_before_device(wq):
    """wq_gemm_grouped checks every linear and the workspace before touching
    the device; its workspace size needs no device."""
    L = wq.lib
    P = 1 << 20

    def lin(N=64, K=1024, group=128, x=P, z=P):
        return wq.Linear(x, P, P, z, P, N, K, group)

    arr = (wq.Linear * 2)(lin(), lin(N=96, K=2048, group=0))
    n1 = L.wq_gemm_grouped_workspace_size(arr, 2, 1, 4)
    n16 = L.wq_gemm_grouped_workspace_size(arr, 2, 16, 4)
    assert 0 < n1 < n16
    assert L.wq_gemm_grouped_workspace_size(arr, 2, 17, 4) == 0          # M > 16: no workspace
    assert L.wq_gemm_grouped_workspace_size(arr, 2, 1, 5) == 0           # bad bits
    small = (wq.Linear * 1)(lin(K=96, group=32))                         # not the persistent kernel's shape
    assert L.wq_gemm_grouped_workspace_size(small, 1, 1, 4) == 0
    assert L.wq_gemm_grouped(arr, 2, 1, 4, None, 0, None) == wq.WQ_ERR_WORKSPACE
    assert L.wq_gemm_grouped(arr, 2, 1, 4, P, n1 - 1, None) == wq.WQ_ERR_WORKSPACE
    assert L.wq_gemm_grouped(arr, 2, 1, 4, P + 8, n1, None) == wq.WQ_ERR_ALIGN
    assert L.wq_gemm_grouped(None, 2, 1, 4, P, n1, None) == wq.WQ_ERR_NULL
    assert L.wq_gemm_grouped(arr, 0, 1, 4, P, n1, None) == wq.WQ_ERR_SHAPE
    assert L.wq_gemm_grouped(arr, 2, 0, 4, P, n1, None) == wq.WQ_ERR_SHAPE
    assert L.wq_gemm_grouped(arr, 2, 1, 7, P, n1, None) == wq.WQ_ERR_BITS
    bad = (wq.Linear * 2)(lin(), lin(group=96))
    assert L.wq_gemm_grouped(bad, 2, 1, 4, P, n1, None) == wq.WQ_ERR_GROUP
    bad = (wq.Linear * 2)(lin(), lin(x=P + 2))
    assert L.wq_gemm_grouped(bad, 2, 1, 4, P, n1, None) == wq.WQ_ERR_ALIGN
    bad = (wq.Linear * 2)(lin(), lin(K=100))
    assert L.wq_gemm_grouped(bad, 2, 1, 4, P, n1, None) == wq.WQ_ERR_SHAPE


def test_symmetric_entry_points_reject_before_device(wq):
    """wq_quantize_rtn_sym checks its arguments like wq_quantize_rtn; a NULL
    zeros pointer is the symmetric grid for wq_gemm, not an error."""
    L = wq.lib
    P = 1 << 20
    q = L.wq_quantize_rtn_sym
    assert q(None, 4, 64, 4, 32, P, P, None) == wq.WQ_ERR_NULL
    assert q(P, 4, 64, 4, 32, P, None, None) == wq.WQ_ERR_NULL
    assert q(P, 4, 64, 6, 32, P, P, None) == wq.WQ_ERR_BITS
    assert q(P, 4, 63, 4, 0, P, P, None) == wq.WQ_ERR_SHAPE
    assert q(P, 4, 64, 4, 48, P, P, None) == wq.WQ_ERR_GROUP
    assert q(P, 4, 64, 4, 32, P + 4, P, None) == wq.WQ_ERR_ALIGN
    g = L.wq_gemm
    st = g(P, 1, 4, 64, P, P, None, 4, 32, P, None)
    assert st not in (wq.WQ_ERR_NULL, wq.WQ_ERR_ALIGN, wq.WQ_ERR_SHAPE, wq.WQ_ERR_GROUP, wq.WQ_ERR_BITS)
    assert g(P, 1, 4, 64, P, None, None, 4, 32, P, None) == wq.WQ_ERR_NULL     # scales are required
    arr = (wq.Linear * 1)(wq.Linear(P, P, P, None, P, 64, 1024, 128))
    assert L.wq_gemm_grouped_workspace_size(arr, 1, 1, 4) > 0
