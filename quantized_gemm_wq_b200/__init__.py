"""Python binding of libwq.so (argument marshalling only).

Every computation happens in the CUDA kernels behind the C ABI declared in
``include/wq.h``; this module only turns torch CUDA tensors into pointers,
allocates outputs with torch (device memory is PyTorch's job here) and raises
``WQError`` on a non-OK status.  There is no fallback: if ``libwq.so`` cannot
be loaded, importing this package fails.

    codes, scales, zeros = wq_quantize_rtn(W_f16, bits, group)
    y = wq_gemm(x_bf16, codes, scales, zeros, bits, group, N, K)
    ys = wq_gemm_grouped([(x, codes, scales, zeros, N, K, group), ...], bits, workspace)
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
WQ_ERR_WORKSPACE = 9

# Functions the header declares (the tests check the library exports them).
EXPORTED = ("wq_quantize_rtn", "wq_quantize_rtn_sym", "wq_gemm", "wq_gemm_grouped", "wq_gemm_grouped_workspace_size",
            "wq_gemm_grouped_noalloc",
            "wq_codes_words", "wq_params_count", "wq_status_string", "wq_last_device_error")


class Linear(ctypes.Structure):
    """``wq_linear`` of include/wq.h: one linear of a grouped call."""
    _fields_ = [("x_bf16", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales_f16", ctypes.c_void_p), ("zeros_f16", ctypes.c_void_p),
                ("y_bf16", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("group", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libwq.so not built ({LIB_PATH}); run __graft_entry__.build() "
                          "or python quantized_gemm_wq_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.wq_quantize_rtn.argtypes = [vp, i64, i64, ci, i64, vp, vp, vp, vp]
    lib.wq_quantize_rtn.restype = ci
    lib.wq_quantize_rtn_sym.argtypes = [vp, i64, i64, ci, i64, vp, vp, vp]
    lib.wq_quantize_rtn_sym.restype = ci
    lib.wq_gemm.argtypes = [vp, i64, i64, i64, vp, vp, vp, ci, i64, vp, vp]
    lib.wq_gemm.restype = ci
    lp = ctypes.POINTER(Linear)
    lib.wq_gemm_grouped.argtypes = [lp, ci, i64, ci, vp, ctypes.c_size_t, vp]
    lib.wq_gemm_grouped.restype = ci
    lib.wq_gemm_grouped_noalloc.argtypes = [lp, ci, i64, ci, vp]
    lib.wq_gemm_grouped_noalloc.restype = ci
    lib.wq_gemm_grouped_workspace_size.argtypes = [lp, ci, i64, ci]
    lib.wq_gemm_grouped_workspace_size.restype = ctypes.c_size_t
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


def wq_quantize_rtn_sym(W: torch.Tensor, bits: int, group: int, codes=None, scales=None, stream=None):
    """Quantise fp16 ``W`` [N, K] (CUDA) on the symmetric grid (zero 2^(bits-1),
    not stored) -> (codes, scales, None); pass the None as ``zeros``."""
    if W.dtype != torch.float16 or W.dim() != 2 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous CUDA fp16 [N, K] tensor")
    N, K = W.shape
    G = groups_per_row(K, group) if group in (0, K) or (group > 0 and K % group == 0) else 1
    if codes is None:
        codes = torch.empty((N, max(1, K * bits // 32)), dtype=torch.int32, device=W.device)
    if scales is None:
        scales = torch.empty((N, G), dtype=torch.float16, device=W.device)
    st = lib.wq_quantize_rtn_sym(_ptr(W), N, K, bits, group, _ptr(codes), _ptr(scales), _stream_ptr(stream))
    _check(st, "wq_quantize_rtn_sym")
    return codes, scales, None


def wq_gemm(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zeros,
            bits: int, group: int, N: int, K: int, y=None, stream=None) -> torch.Tensor:
    """``y = x . W'^T`` for bf16 ``x`` [M, K] (CUDA) -> bf16 ``y`` [M, N];
    ``zeros`` None for codes of the symmetric grid."""
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


def _linear_array(items, M):
    """ctypes array of ``wq_linear`` from (x, codes, scales, zeros, N, K, group, y)
    tuples; allocates the missing outputs."""
    arr = (Linear * len(items))()
    ys = []
    for i, it in enumerate(items):
        x, codes, scales, zeros, N, K, group = it[:7]
        y = it[7] if len(it) > 7 and it[7] is not None else None
        if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or not x.is_contiguous():
            raise ValueError("every x must be a contiguous CUDA bf16 [M, K] tensor")
        if x.shape[0] != M or x.shape[1] != K:
            raise ValueError("every x must be [M, K] with the call's M")
        if y is None:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        arr[i] = Linear(_ptr(x), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(y), N, K, group)
        ys.append(y)
    return arr, ys


def grouped_workspace_size(items, bits: int) -> int:
    """Workspace bytes ``wq_gemm_grouped`` needs for these linears."""
    if not items:
        return 0
    M = items[0][0].shape[0]
    arr, _ = _linear_array([it[:7] for it in items], M) if items[0][0].is_cuda else (None, None)
    if arr is None:
        raise ValueError("x must be a CUDA tensor")
    return int(lib.wq_gemm_grouped_workspace_size(arr, len(items), M, bits))


def grouped_workspace(items, bits: int, device=None) -> torch.Tensor:
    """A zero-filled device workspace for ``wq_gemm_grouped`` on these linears
    (uint8, at least 16 bytes so it always has an address)."""
    n = grouped_workspace_size(items, bits)
    dev = device if device is not None else items[0][0].device
    return torch.zeros(max(16, n), dtype=torch.uint8, device=dev)


def wq_gemm_grouped(items, bits: int, workspace=None, stream=None):
    """``y_l = x_l . W'_l^T`` for every (x, codes, scales, zeros, N, K, group[, y])
    of ``items`` (common M and bits) -> list of bf16 ``y_l``.  ``workspace``: a
    zero-filled uint8 CUDA tensor from ``grouped_workspace`` (made here when
    None; reuse one across calls on the same stream)."""
    if not items:
        return []
    M = items[0][0].shape[0]
    arr, ys = _linear_array(items, M)
    if workspace is None:
        workspace = grouped_workspace(items, bits)
    st = lib.wq_gemm_grouped(arr, len(items), M, bits, _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check(st, "wq_gemm_grouped")
    return ys


def wq_gemm_grouped_noalloc(items, bits: int, stream=None):
    """``wq_gemm_grouped`` on the library's built-in 8 MiB workspace, for
    callers that cannot allocate device memory when they call.  Every item
    must carry its output ``y`` (x, codes, scales, zeros, N, K, group, y):
    nothing is allocated here either."""
    if not items:
        return []
    if any(len(it) < 8 or it[7] is None for it in items):
        raise ValueError("wq_gemm_grouped_noalloc allocates nothing: pass every y")
    M = items[0][0].shape[0]
    arr, ys = _linear_array(items, M)
    st = lib.wq_gemm_grouped_noalloc(arr, len(items), M, bits, _stream_ptr(stream))
    _check(st, "wq_gemm_grouped_noalloc")
    return ys
