"""Python binding of libwq.so (argument marshalling only).

Every computation happens in the CUDA kernels behind the C ABI declared in
``include/wq.h``; this module only turns torch CUDA tensors into pointers,
allocates outputs with torch (device memory is PyTorch's job here) and raises
``WQError`` on a non-OK status.  There is no fallback: if ``libwq.so`` cannot
be loaded, importing this package fails.

    codes, scales, zeros = wq_quantize_rtn(W_f16, bits, group)
    y = wq_gemm(x_bf16, codes, scales, zeros, bits, group, N, K)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwq.so")

# Status codes of include/wq.h
WQ_OK = 0
WQ_ERR_NULL = 1
WQ_ERR_BITS = 2
WQ_ERR_GROUP = 3
WQ_ERR_SHAPE = 4
WQ_ERR_ALIGN = 5
WQ_ERR_UNSUPPORTED_DEVICE = 6
WQ_ERR_CUDA = 7
WQ_ERR_DEVICE_TIMEOUT = 8

# Functions the header declares (the tests check the library exports them).
EXPORTED = ("wq_quantize_rtn", "wq_gemm", "wq_codes_words", "wq_params_count",
            "wq_status_string", "wq_last_device_error")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libwq.so not built ({LIB_PATH}); run __graft_entry__.build() "
                          "or python quantized_gemm_wq_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.wq_quantize_rtn.argtypes = [vp, i64, i64, ci, i64, vp, vp, vp, vp]
    lib.wq_quantize_rtn.restype = ci
    lib.wq_gemm.argtypes = [vp, i64, i64, i64, vp, vp, vp, ci, i64, vp, vp]
    lib.wq_gemm.restype = ci
    lib.wq_codes_words.argtypes = [i64, i64, ci]
    lib.wq_codes_words.restype = ctypes.c_size_t
    lib.wq_params_count.argtypes = [i64, i64, i64]
    lib.wq_params_count.restype = ctypes.c_size_t
    lib.wq_status_string.argtypes = [ci]
    lib.wq_status_string.restype = ctypes.c_char_p
    lib.wq_last_device_error.argtypes = []
    lib.wq_last_device_error.restype = ci
    return lib


lib = _load()


class WQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.wq_status_string(status).decode()} (status {status})")


def _check(status: int, where: str) -> None:
    if status != WQ_OK:
        raise WQError(status, where)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def wq_codes_words(N: int, K: int, bits: int) -> int:
    return int(lib.wq_codes_words(N, K, bits))


def wq_params_count(N: int, K: int, group: int) -> int:
    return int(lib.wq_params_count(N, K, group))


def wq_status_string(status: int) -> str:
    return lib.wq_status_string(status).decode()


def wq_last_device_error() -> int:
    return int(lib.wq_last_device_error())


def groups_per_row(K: int, group: int) -> int:
    return 1 if group in (0, K) else K // group


def wq_quantize_rtn(W: torch.Tensor, bits: int, group: int, codes=None, scales=None,
                    zeros=None, stream=None):
    """Quantise fp16 ``W`` [N, K] (CUDA) -> (codes uint32 [N, K*bits/32] as
    int32 storage, scales fp16 [N, G], zeros fp16 [N, G])."""
    if W.dtype != torch.float16 or W.dim() != 2 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous CUDA fp16 [N, K] tensor")
    N, K = W.shape
    G = groups_per_row(K, group) if group in (0, K) or (group > 0 and K % group == 0) else 1
    if codes is None:
        codes = torch.empty((N, max(1, K * bits // 32)), dtype=torch.int32, device=W.device)
    if scales is None:
        scales = torch.empty((N, G), dtype=torch.float16, device=W.device)
    if zeros is None:
        zeros = torch.empty((N, G), dtype=torch.float16, device=W.device)
    st = lib.wq_quantize_rtn(_ptr(W), N, K, bits, group, _ptr(codes), _ptr(scales), _ptr(zeros),
                             _stream_ptr(stream))
    _check(st, "wq_quantize_rtn")
    return codes, scales, zeros


def wq_gemm(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
            bits: int, group: int, N: int, K: int, y=None, stream=None) -> torch.Tensor:
    """``y = x . W'^T`` for bf16 ``x`` [M, K] (CUDA) -> bf16 ``y`` [M, N]."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA bf16 [M, K] tensor")
    M = x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x.shape[1] must equal K")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    st = lib.wq_gemm(_ptr(x), M, N, K, _ptr(codes), _ptr(scales), _ptr(zeros), bits, group,
                     _ptr(y), _stream_ptr(stream))
    _check(st, "wq_gemm")
    return y
