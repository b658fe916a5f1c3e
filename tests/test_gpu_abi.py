"""The C ABI's contract on a real device (include/wq.h, "Common rules for the
compute calls"): a call that returns a failing status has launched nothing and
written no byte of any output buffer, and the work of a successful call runs on
the stream it was given.

Failing calls go straight through ctypes to libwq.so with real device buffers
filled with a canary pattern, so the binding's own argument checks are not what
is being tested."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import wq_inputs
from gpu_util import wq

pytestmark = pytest.mark.gpu

CANARY = 0x5A


def _canary(shape, dtype):
    t = torch.empty(shape, dtype=dtype, device="cuda")
    t.view(torch.uint8).fill_(CANARY)
    return t


def _untouched(*ts):
    torch.cuda.synchronize()
    for t in ts:
        b = t.contiguous().view(torch.uint8).cpu().numpy()
        assert np.all(b == CANARY), f"{int((b != CANARY).sum())} bytes written by a failing call"


def _quantized(N, K, bits, group, seed=0):
    Wh = wq_inputs.weight_f16(seed, 0, N, K)
    return wq().wq_quantize_rtn(torch.from_numpy(Wh).cuda(), bits, group)


def test_failing_quantize_writes_nothing():
    m = wq()
    N, K = 256, 1024
    W = torch.from_numpy(wq_inputs.weight_f16(0, 0, N, K)).cuda()
    codes = _canary((N, K * 4 // 32), torch.int32)
    s = _canary((N, K // 128), torch.float16)
    z = _canary((N, K // 128), torch.float16)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    cases = [
        (dict(bits=5, group=128), m.WQ_ERR_BITS),
        (dict(bits=4, group=48), m.WQ_ERR_GROUP),    # not a multiple of 32
        (dict(bits=4, group=96), m.WQ_ERR_GROUP),    # does not divide K
    ]
    for kw, want in cases:
        st = m.lib.wq_quantize_rtn(p(W), N, K, kw["bits"], kw["group"], p(codes), p(s), p(z), None)
        assert st == want, (kw, st)
    # a misaligned output pointer (4 bytes into the buffer)
    st = m.lib.wq_quantize_rtn(p(W), N, K, 4, 128, ctypes.c_void_p(codes.data_ptr() + 4), p(s), p(z), None)
    assert st == m.WQ_ERR_ALIGN
    _untouched(codes, s, z)
    st = m.lib.wq_quantize_rtn_sym(p(W), N, K, 4, 100, p(codes), p(s), None)
    assert st == m.WQ_ERR_GROUP
    _untouched(codes, s)


@pytest.mark.parametrize("M", [1, 4, 16, 64, 300])
def test_failing_gemm_writes_nothing(M):
    """Every batch size reaches a different kernel on success; on a failing
    status none of them may have run."""
    m = wq()
    N, K, bits, group = 512, 1024, 4, 128
    codes, s, z = _quantized(N, K, bits, group)
    x = wq_inputs.activations_bf16(0, 1, M, K).cuda()
    y = _canary((M, N), torch.bfloat16)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    bad = [
        ((p(x), M, N, K, p(codes), p(s), p(z), 6, group, p(y), None), m.WQ_ERR_BITS),
        ((p(x), M, N, K, p(codes), p(s), p(z), bits, 80, p(y), None), m.WQ_ERR_GROUP),
        ((p(x), M, N, K + 16, p(codes), p(s), p(z), bits, group, p(y), None), m.WQ_ERR_SHAPE),   # K % 32
        ((p(x), M, N, K, None, p(s), p(z), bits, group, p(y), None), m.WQ_ERR_NULL),
        ((p(x), M, N, K, p(codes), p(s), p(z), bits, group, ctypes.c_void_p(y.data_ptr() + 2), None),
         m.WQ_ERR_ALIGN),
        ((ctypes.c_void_p(x.data_ptr() + 8), M, N, K, p(codes), p(s), p(z), bits, group, p(y), None),
         m.WQ_ERR_ALIGN),
    ]
    for args, want in bad:
        st = m.lib.wq_gemm(*args)
        assert st == want, (want, st)
    _untouched(y)


def test_failing_grouped_writes_nothing():
    """A grouped call whose second linear is invalid, or whose workspace is
    too small, writes neither linear's y (all checks precede every launch)."""
    m = wq()
    M, bits, group = 4, 4, 128
    items = []
    for i, (N, K) in enumerate([(384, 1024), (256, 2048)]):
        c, s, z = _quantized(N, K, bits, group, seed=i)
        x = wq_inputs.activations_bf16(i, 1, M, K).cuda()
        items.append((x, c, s, z, N, K, group, _canary((M, N), torch.bfloat16)))
    ws = m.grouped_workspace([it[:7] for it in items], bits)
    arr, ys = m._linear_array(items, M)
    # second linear with a group that does not divide K
    arr[1].group = 96 * 4
    nbytes = ws.numel()
    st = m.lib.wq_gemm_grouped(arr, 2, M, bits, ctypes.c_void_p(ws.data_ptr()), nbytes, None)
    assert st == m.WQ_ERR_GROUP
    arr[1].group = group
    # workspace one byte short
    need = m.lib.wq_gemm_grouped_workspace_size(arr, 2, M, bits)
    assert need > 0
    st = m.lib.wq_gemm_grouped(arr, 2, M, bits, ctypes.c_void_p(ws.data_ptr()), need - 1, None)
    assert st == m.WQ_ERR_WORKSPACE
    _untouched(*ys)
    # and the same call with a valid workspace succeeds and writes both
    st = m.lib.wq_gemm_grouped(arr, 2, M, bits, ctypes.c_void_p(ws.data_ptr()), nbytes, None)
    assert st == m.WQ_OK
    torch.cuda.synchronize()
    for y in ys:
        assert not np.all(y.view(torch.uint8).cpu().numpy() == CANARY)


@pytest.mark.parametrize("M", [1, 4, 64])
def test_gemm_runs_on_the_given_stream(M):
    """Work queued behind a long sleep on a side stream has not run when the
    default stream is drained, and has run once the side stream is."""
    m = wq()
    N, K, bits, group = 512, 1024, 4, 128
    codes, s, z = _quantized(N, K, bits, group)
    x = wq_inputs.activations_bf16(0, 1, M, K).cuda()
    y = _canary((M, N), torch.bfloat16)
    ref = m.wq_gemm(x, codes, s, z, bits, group, N, K)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        torch.cuda._sleep(200_000_000)          # ~0.1 s of device time on `side`
    m.wq_gemm(x, codes, s, z, bits, group, N, K, y=y, stream=side)
    done = torch.cuda.Event()
    done.record(side)
    torch.cuda.current_stream().synchronize()
    early = y.view(torch.uint8).cpu().numpy()   # read on the default stream
    assert not done.query(), "the side stream finished before the check; sleep too short"
    assert np.all(early == CANARY), "wq_gemm ran before the work queued ahead of it on its stream"
    side.synchronize()
    assert torch.equal(y, ref)


def test_grouped_runs_on_the_given_stream():
    m = wq()
    M, bits, group = 1, 4, 128
    items = []
    for i, (N, K) in enumerate([(384, 1024), (256, 2048)]):
        c, s, z = _quantized(N, K, bits, group, seed=i)
        x = wq_inputs.activations_bf16(i, 1, M, K).cuda()
        items.append((x, c, s, z, N, K, group, _canary((M, N), torch.bfloat16)))
    ws = m.grouped_workspace(items, bits)
    refs = m.wq_gemm_grouped([it[:7] for it in items], bits)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        torch.cuda._sleep(200_000_000)
    ys = m.wq_gemm_grouped(items, bits, workspace=ws, stream=side)
    done = torch.cuda.Event()
    done.record(side)
    torch.cuda.current_stream().synchronize()
    early = [y.view(torch.uint8).cpu().numpy() for y in ys]
    assert not done.query()
    assert all(np.all(e == CANARY) for e in early)
    side.synchronize()
    for y, r in zip(ys, refs):
        assert torch.equal(y, r)
