"""CPU oracle for the weight-only quantised GEMM (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  The C++
source (``wq_oracle.cpp``) states the method and the readings it takes; every
function here only marshals numpy arrays.

Parity status of each function (what pins it, see ``tests/test_oracle.py``):

* ``f16_to_f64`` / ``f64_to_f16`` / ``bf16_to_f64`` / ``f64_to_bf16``: pinned
  (exhaustive decode against IEEE definitions via numpy/torch casts, RNE
  midpoints by exact arithmetic).
* ``quantize_rtn``: pinned (closed-form designed grids, brute-force nearest grid
  point in exact rational arithmetic, exact rational scale/zero, invariants).
* ``quantize_rtn_sym``: pinned (designed symmetric grids, brute-force nearest
  grid point in exact rational arithmetic, exact rational scale, odd symmetry,
  invariants).
* ``pack`` / ``unpack``: pinned (hand-derived words in ``tests/golden``,
  round trips).
* ``dequant`` / ``gemm``: pinned (exact rational sums on tiny inputs, one-hot
  and zero inputs, permutation invariance).
* ``hessian`` / ``quantize_optq``: pinned (``tests/test_oracle_optq.py``): the
  compensated weights at every step against the least-squares re-fit solved by
  ``numpy.linalg.solve``; a diagonal Hessian reproduces ``quantize_rtn`` bit for
  bit; a factor 4 on H changes nothing; the first column of every row and the
  first group's grid equal round-to-nearest's; the layer's output error on the
  calibration rows falls below round-to-nearest's.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        for name in ("orc_f16_to_f64", "orc_f64_to_f16", "orc_bf16_to_f64", "orc_f64_to_bf16"):
            getattr(lib, name).argtypes = [_p, _p, _i64]
            getattr(lib, name).restype = None
        lib.orc_quantize_rtn.argtypes = [_p, _i64, _i64, ctypes.c_int, _i64, _p, _p, _p, ctypes.c_int]
        lib.orc_quantize_rtn.restype = ctypes.c_int
        lib.orc_quantize_rtn_sym.argtypes = [_p, _i64, _i64, ctypes.c_int, _i64, _p, _p, ctypes.c_int]
        lib.orc_quantize_rtn_sym.restype = ctypes.c_int
        lib.orc_quantize_optq.argtypes = [_p, _p, _i64, _i64, ctypes.c_int, _i64, ctypes.c_double,
                                          _p, _p, _p, _p, ctypes.c_int]
        lib.orc_quantize_optq.restype = ctypes.c_int
        lib.orc_pack.argtypes = [_p, _i64, _i64, ctypes.c_int, _p]
        lib.orc_pack.restype = ctypes.c_int
        lib.orc_unpack.argtypes = [_p, _i64, _i64, ctypes.c_int, _p]
        lib.orc_unpack.restype = ctypes.c_int
        lib.orc_dequant.argtypes = [_p, _p, _p, _i64, _i64, _i64, _p]
        lib.orc_dequant.restype = ctypes.c_int
        lib.orc_gemm.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, ctypes.c_int, _i64,
                                 _p, _i64, _p, _p, ctypes.c_int]
        lib.orc_gemm.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(ValueError):
    pass


def groups_per_row(K: int, group: int) -> int:
    return 1 if group in (0, K) else K // group


def words_per_row(K: int, bits: int) -> int:
    return K * bits // 32


def f16_to_f64(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    _lib().orc_f16_to_f64(_ptr(h), _ptr(out), h.size)
    return out


def f64_to_f16(d):
    d = _c(d, np.float64)
    out = np.empty(d.shape, np.uint16)
    _lib().orc_f64_to_f16(_ptr(d), _ptr(out), d.size)
    return out


def bf16_to_f64(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    _lib().orc_bf16_to_f64(_ptr(h), _ptr(out), h.size)
    return out


def f64_to_bf16(d):
    d = _c(d, np.float64)
    out = np.empty(d.shape, np.uint16)
    _lib().orc_f64_to_bf16(_ptr(d), _ptr(out), d.size)
    return out


def quantize_rtn(W_bits, bits: int, group: int, nthreads: int = 0):
    """Round-to-nearest quantisation of fp16 ``W`` (uint16 bit patterns [N, K]).

    Returns ``(q, scales, zeros)``: unpacked codes uint8 [N, K] and fp16 bit
    patterns uint16 [N, G]."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    G = groups_per_row(K, group) if K % 32 == 0 and (group in (0, K) or (group > 0 and K % group == 0)) else 1
    q = np.empty((N, K), np.uint8)
    s = np.empty((N, G), np.uint16)
    z = np.empty((N, G), np.uint16)
    rc = _lib().orc_quantize_rtn(_ptr(W), N, K, bits, group, _ptr(q), _ptr(s), _ptr(z), nthreads)
    if rc != 0:
        raise OracleError(f"invalid arguments N={N} K={K} bits={bits} group={group}")
    return q, s, z


def quantize_rtn_sym(W_bits, bits: int, group: int, nthreads: int = 0):
    """Round-to-nearest quantisation on the symmetric grid (zero fixed at
    2^(bits-1), not stored).  Returns ``(q, scales)``."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    G = groups_per_row(K, group) if K % 32 == 0 and (group in (0, K) or (group > 0 and K % group == 0)) else 1
    q = np.empty((N, K), np.uint8)
    s = np.empty((N, G), np.uint16)
    rc = _lib().orc_quantize_rtn_sym(_ptr(W), N, K, bits, group, _ptr(q), _ptr(s), nthreads)
    if rc != 0:
        raise OracleError(f"invalid arguments N={N} K={K} bits={bits} group={group}")
    return q, s


def hessian(x_bits):
    """Layer Hessian of calibration activations (reading O1 of the C++
    source): ``H = (2 / S) X^T X`` in fp64 for bf16 bit patterns ``x_bits``
    [S, K]."""
    X = bf16_to_f64(x_bits)
    return (2.0 / X.shape[0]) * (X.T @ X)


def quantize_optq(W_bits, H, bits: int, group: int, percdamp: float = 0.01,
                  return_u: bool = False, nthreads: int = 0):
    """Error-compensating quantisation of fp16 ``W`` (uint16 bit patterns
    [N, K]) against the layer Hessian ``H`` (fp64 [K, K]).

    Returns ``(q, scales, zeros)`` like ``quantize_rtn`` and, with
    ``return_u``, the fp64 weights [N, K] as each column came up."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    Hc = _c(H, np.float64)
    if Hc.shape != (K, K):
        raise OracleError("H must be [K, K]")
    G = 1 if group in (0, K) else (K // group if group > 0 and K % group == 0 else 1)
    q = np.empty((N, K), np.uint8)
    s = np.empty((N, G), np.uint16)
    z = np.empty((N, G), np.uint16)
    u = np.empty((N, K), np.float64) if return_u else None
    rc = _lib().orc_quantize_optq(_ptr(W), _ptr(Hc), N, K, bits, group, float(percdamp),
                                  _ptr(q), _ptr(s), _ptr(z), _ptr(u) if return_u else None,
                                  nthreads)
    if rc == -2:
        raise OracleError("the damped Hessian is not positive definite")
    if rc != 0:
        raise OracleError(f"invalid arguments N={N} K={K} bits={bits} group={group}")
    return (q, s, z, u) if return_u else (q, s, z)


def sym_zeros(scales, bits: int):
    """The zeros a symmetric grid implies: fp16 bit patterns of 2^(bits-1), the
    shape of ``scales`` (what ``dequant`` and ``gemm`` take)."""
    s = np.asarray(scales)
    return np.full(s.shape, f64_to_f16(np.array([float(1 << (bits - 1))]))[0], np.uint16)


def pack(q, bits: int):
    q = _c(q, np.uint8)
    N, K = q.shape
    w = np.empty((N, words_per_row(K, bits)), np.uint32)
    if _lib().orc_pack(_ptr(q), N, K, bits, _ptr(w)) != 0:
        raise OracleError("invalid pack arguments")
    return w


def unpack(words, K: int, bits: int):
    w = _c(words, np.uint32)
    N = w.shape[0]
    if w.shape[1] != words_per_row(K, bits):
        raise OracleError("word count does not match K and bits")
    q = np.empty((N, K), np.uint8)
    if _lib().orc_unpack(_ptr(w), N, K, bits, _ptr(q)) != 0:
        raise OracleError("invalid unpack arguments")
    return q


def dequant(q, scales, zeros, group: int):
    q = _c(q, np.uint8)
    s = _c(scales, np.uint16)
    z = _c(zeros, np.uint16)
    N, K = q.shape
    out = np.empty((N, K), np.float64)
    if _lib().orc_dequant(_ptr(q), _ptr(s), _ptr(z), N, K, group, _ptr(out)) != 0:
        raise OracleError("invalid dequant arguments")
    return out


def gemm(x_bits, words, scales, zeros, N: int, K: int, bits: int, group: int,
         cols=None, nthreads: int = 0):
    """fp64 ``y = x . W'^T`` and ``bound = sum_k |x w'|`` for the output
    columns ``cols`` (all N when None).  ``x_bits``: bf16 bit patterns [M, K]."""
    x = _c(x_bits, np.uint16)
    M = x.shape[0]
    w = _c(words, np.uint32)
    s = _c(scales, np.uint16)
    z = _c(zeros, np.uint16)
    if cols is None:
        ncols = N
        cp = None
    else:
        cols = _c(cols, np.int64)
        ncols = cols.size
        cp = _ptr(cols)
    y = np.empty((M, ncols), np.float64)
    b = np.empty((M, ncols), np.float64)
    rc = _lib().orc_gemm(_ptr(x), M, N, K, _ptr(w), _ptr(s), _ptr(z), bits, group, cp, ncols,
                         _ptr(y), _ptr(b), nthreads)
    if rc != 0:
        raise OracleError("invalid gemm arguments")
    return y, b
