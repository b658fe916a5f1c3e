"""Bounded device waits (failure handling without a GPU fault).

libwq_shortwait.so is the test build of the library: pipeline-wait limit 0 and
one test hook, wq_test_expire_wait, a kernel whose bounded wait is on an
mbarrier that nothing arrives on.  In a child process:
  * the hook's wait runs out and wq_last_device_error reports
    WQ_ERR_DEVICE_TIMEOUT once (a second read finds the flag cleared);
  * the decode kernels of that build (M = 1 GEMV, 2..8-token warp-MMA GEMV,
    grouped GEMV) run with a zero limit: each wait either finds its stage
    landed or gives up, drains its copies and leaves;
  * right after, in the same process and context, the normal library computes
    y correctly and reports no expired wait."""
from __future__ import annotations

import ctypes
import multiprocessing as mp
import os

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _child(q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    try:
        import numpy as np
        import torch

        import oracle
        import quantized_gemm_wq_b200 as wq
        import wq_inputs
        from gpu_util import assert_y_close, oracle_quantize
        short = ctypes.CDLL(os.path.join(ROOT, "quantized_gemm_wq_b200", "libwq_shortwait.so"))
        i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        short.wq_gemm.argtypes = [vp, i64, i64, i64, vp, vp, vp, ci, i64, vp, vp]
        short.wq_gemm.restype = ci
        short.wq_gemm_grouped.argtypes = [ctypes.POINTER(wq.Linear), ci, i64, ci, vp, ctypes.c_size_t, vp]
        short.wq_gemm_grouped.restype = ci
        short.wq_last_device_error.restype = ci
        short.wq_test_expire_wait.argtypes = [vp]
        short.wq_test_expire_wait.restype = ci
        res = {}
        res["probe_launch"] = short.wq_test_expire_wait(None)
        res["probe_status"] = short.wq_last_device_error()
        res["probe_cleared"] = short.wq_last_device_error()
        N, K, bits, group = 96, 2048, 4, 128
        Wh = wq_inputs.weight_f16(60, 0, N, K)
        c, s, z = wq.wq_quantize_rtn(torch.from_numpy(Wh).cuda(), bits, group)
        for M in (1, 4):
            x = wq_inputs.activations_bf16(60, M, M, K).cuda()
            y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            st = short.wq_gemm(x.data_ptr(), M, N, K, c.data_ptr(), s.data_ptr(), z.data_ptr(), bits, group,
                               y.data_ptr(), None)
            res[f"launch_M{M}"] = st
            res[f"timeout_M{M}"] = short.wq_last_device_error()
        x = wq_inputs.activations_bf16(60, 1, 1, K).cuda()
        y = torch.empty(1, N, dtype=torch.bfloat16, device="cuda")
        items = [(x, c, s, z, N, K, group, y)]
        ws = wq.grouped_workspace(items, bits)
        arr = (wq.Linear * 1)(wq.Linear(x.data_ptr(), c.data_ptr(), s.data_ptr(), z.data_ptr(), y.data_ptr(),
                                       N, K, group))
        res["launch_grouped"] = short.wq_gemm_grouped(arr, 1, 1, bits, ws.data_ptr(), ws.numel(), None)
        res["timeout_grouped"] = short.wq_last_device_error()
        res["second_read_clears"] = short.wq_last_device_error()
        # the normal build, same process and context: correct results, no expired wait
        oc, os_, oz = oracle_quantize(Wh, bits, group)
        for M in (1, 4):
            xc = wq_inputs.activations_bf16(61, M, M, K)
            yg = wq.wq_gemm(xc.cuda(), c, s, z, bits, group, N, K).float().cpu().numpy()
            y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(xc), oc, os_, oz, N, K, bits, group)
            assert_y_close(yg, y_ref, bound, f"normal build after timeouts, M={M}")
        ws.zero_()
        (yg,) = wq.wq_gemm_grouped([(x, c, s, z, N, K, group)], bits, workspace=ws)
        y_ref, bound = oracle.gemm(wq_inputs.bf16_bits(x.cpu()), oc, os_, oz, N, K, bits, group)
        assert_y_close(yg.float().cpu().numpy(), y_ref, bound, "normal build grouped after timeouts")
        res["normal_after"] = wq.wq_last_device_error()
        q.put(("ok", res))
    except Exception as e:  # noqa: BLE001 - reported to the parent
        q.put(("error", repr(e)))


def test_expired_waits_are_reported_and_the_context_survives():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_child, args=(q,))
    p.start()
    kind, res = q.get(timeout=300)
    p.join(timeout=60)
    assert kind == "ok", res
    assert p.exitcode == 0
    assert res["probe_launch"] == 0, res
    assert res["probe_status"] == 8, res                     # WQ_ERR_DEVICE_TIMEOUT
    assert res["probe_cleared"] == 0, res
    for k in ("launch_M1", "launch_M4", "launch_grouped"):
        assert res[k] == 0, (k, res)                         # the launches themselves succeed
    for k in ("timeout_M1", "timeout_M4", "timeout_grouped"):
        assert res[k] in (0, 8), (k, res)                    # done, or gave up and reported it
    assert res["second_read_clears"] == 0
    assert res["normal_after"] == 0
