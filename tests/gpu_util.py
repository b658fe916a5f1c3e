"""Helpers shared by the GPU parity tests: run the library through its C ABI,
run the oracle on the same host bytes, compare."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
import wq_inputs

# Per-element bound on |y_gpu - y_exact| (the accuracy contract of wq_gemm):
# the arithmetic before the output rounding may err by REL_TOL * sum_k |x w'|
# plus an absolute floor, and y itself is bf16, whose round-to-nearest adds up
# to 2^-8 |y| even when every earlier step is exact.
REL_TOL = 2e-3
ABS_TOL = 1e-3
OUT_ROUND = 2.0 ** -8


def wq():
    import quantized_gemm_wq_b200 as m
    return m


def to_dev_f16(Wh: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(Wh)).cuda()


def gpu_quantize(Wh: np.ndarray, bits: int, group: int):
    W = to_dev_f16(Wh)
    codes, s, z = wq().wq_quantize_rtn(W, bits, group)
    torch.cuda.synchronize()
    return (codes.cpu().numpy().view(np.uint32), s.cpu().numpy().view(np.uint16),
            z.cpu().numpy().view(np.uint16))


def oracle_quantize(Wh: np.ndarray, bits: int, group: int):
    q, s, z = oracle.quantize_rtn(wq_inputs.f16_bits(Wh), bits, group)
    return oracle.pack(q, bits), s, z


# Largest max |y - y_ref| / sum_k |x w'| seen by assert_y_close in this run,
# and the largest share of the per-element tolerance used, each with the check
# that produced it (printed in the pytest summary).
WORST = {"ratio": 0.0, "what": "", "used": 0.0, "used_what": ""}


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what: str = ""):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    lim = REL_TOL * bound + OUT_ROUND * np.abs(y_ref) + ABS_TOL
    bad = err > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first "
                             f"{tuple(i)} gpu={y_gpu[tuple(i)]} ref={y_ref[tuple(i)]} "
                             f"bound={bound[tuple(i)]}")
    ratio = float((err / np.maximum(bound, 1e-30)).max()) if err.size else 0.0
    used = float((err / lim).max()) if err.size else 0.0
    if ratio > WORST["ratio"]:
        WORST["ratio"], WORST["what"] = ratio, what
    if used > WORST["used"]:
        WORST["used"], WORST["used_what"] = used, what
    return ratio


@functools.lru_cache(maxsize=8)
def cached_weight(seed, tid, N, K, dist):
    return wq_inputs.weight_f16(seed, tid, N, K, dist=dist)
