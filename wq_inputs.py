"""Seeded synthetic inputs shared by the oracle checks and the CUDA path.

This module holds none of the method's arithmetic: it only draws random
numbers (mixing latent factors into correlated features for the calibration
rows) and casts them to the storage types (fp16 weights, bf16 activations),
so the oracle (``oracle/``) and the library (``quantized_gemm_wq_b200``) are
handed the very same bytes.

Recipe (the pages print no workload data, so the synthetic shapes below stand
in for real checkpoints):

* weights ``W`` fp16 ``[N, K]``: ``0.02 * N(0, 1)`` or, for the heavy-tailed
  OPT-175B-shaped layers, ``0.02 * Student-t(nu=4)``; drawn in float32
  (normal) / float64 (t) by numpy's PCG64 ``default_rng``, then rounded to
  fp16 by numpy (round-to-nearest-even).  Rows are drawn in blocks of
  ``ROW_BLOCK`` rows, each block from its own stream keyed by
  ``(seed, tensor_id, block)``, so any subset of rows can be regenerated
  without drawing the whole matrix.
* activations ``x`` bf16 ``[M, K]``: ``N(0, 1)`` drawn in float32 per row
  stream ``(seed, tensor_id, 1_000_000 + m)`` and rounded to bf16 by torch's
  CPU cast (round-to-nearest-even).

* calibration activations bf16 ``[S, K]`` (stand-in for the pages' 128
  segments of 2048 tokens of C4 text): correlated features with a few
  outlier channels, ``x = c * (z + lam @ f)`` with ``z ~ N(0, I_K)``,
  ``RANK`` latent factors ``f ~ N(0, I)`` per row, loadings
  ``lam ~ N(0, 1/RANK)`` per feature, and per-feature scales ``c`` = 1 except
  ``OUTLIER_FRAC`` of the features at ``OUTLIER_SCALE``; drawn in float64 from
  one stream keyed by ``(seed, tensor_id, 2_000_000)``, rounded to bf16 by
  torch's CPU cast.

The workload table ``WORKLOADS`` lists the five single-GPU configurations the
library is tested and measured on (shapes of a single 4096x4096 linear, a
Llama-7B-shaped decoder layer, OPT-175B-shaped FC1/FC2, Llama-13B-shaped
prefill GEMMs and a 32-layer 7B-shaped stack).
"""
from __future__ import annotations

import numpy as np
import torch

ROW_BLOCK = 256


def _row_block_stream(seed: int, tensor_id: int, block: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id), int(block)])


def weight_f16(seed: int, tensor_id: int, N: int, K: int, dist: str = "normal",
               scale: float = 0.02, rows=None) -> np.ndarray:
    """fp16 weight matrix ``[N, K]`` (or only ``rows`` of it, in that order)."""
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= N):
        raise ValueError("row index out of range")
    out = np.empty((rows.size, K), dtype=np.float16)
    blocks = np.unique(rows // ROW_BLOCK)
    for b in blocks:
        r0 = int(b) * ROW_BLOCK
        nb = min(ROW_BLOCK, N - r0)
        g = _row_block_stream(seed, tensor_id, int(b))
        if dist == "normal":
            v = g.standard_normal((nb, K), dtype=np.float32) * np.float32(scale)
        elif dist == "t4":
            v = g.standard_t(4.0, size=(nb, K)) * scale
        else:
            raise ValueError(f"unknown distribution {dist!r}")
        blk = v.astype(np.float16)
        sel = np.nonzero(rows // ROW_BLOCK == b)[0]
        out[sel] = blk[rows[sel] - r0]
    return out


def activations_bf16(seed: int, tensor_id: int, M: int, K: int) -> torch.Tensor:
    """bf16 activation matrix ``[M, K]`` on the CPU, entries ``N(0, 1)``."""
    v = np.empty((M, K), dtype=np.float32)
    for m in range(M):
        g = np.random.default_rng([int(seed), int(tensor_id), 1_000_000 + m])
        v[m] = g.standard_normal(K, dtype=np.float32)
    return torch.from_numpy(v).to(torch.bfloat16)


CALIB_RANK = 16
CALIB_OUTLIER_FRAC = 0.02
CALIB_OUTLIER_SCALE = 20.0


def calibration_bf16(seed: int, tensor_id: int, S: int, K: int) -> torch.Tensor:
    """bf16 calibration activations ``[S, K]`` on the CPU (recipe above)."""
    g = np.random.default_rng([int(seed), int(tensor_id), 2_000_000])
    lam = g.standard_normal((CALIB_RANK, K)) / np.sqrt(CALIB_RANK)
    c = np.ones(K)
    n_out = max(1, int(round(CALIB_OUTLIER_FRAC * K)))
    c[g.choice(K, n_out, replace=False)] = CALIB_OUTLIER_SCALE
    f = g.standard_normal((S, CALIB_RANK))
    z = g.standard_normal((S, K))
    v = (z + f @ lam) * c
    return torch.from_numpy(v).to(torch.bfloat16)


def f16_bits(a: np.ndarray) -> np.ndarray:
    """View an fp16 array as its uint16 bit patterns."""
    return np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """View a bf16 tensor as its uint16 bit patterns (numpy)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# Workloads.  Each linear is (name, N, K); y = x . W'^T with x [M, K].
# ---------------------------------------------------------------------------
LLAMA7B_LAYER = [("qkv", 12288, 4096), ("o", 4096, 4096),
                 ("gate_up", 22016, 4096), ("down", 4096, 11008)]
LLAMA7B_STACK_LAYER = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096),
                       ("o", 4096, 4096), ("gate", 11008, 4096), ("up", 11008, 4096),
                       ("down", 4096, 11008)]

WORKLOADS = {
    "linear4096_4b_g128": dict(
        desc="single linear 4096x4096, 4-bit, group 128, W~N(0,0.02^2), x [1,4096]",
        linears=[("linear", 4096, 4096)], bits=4, group=128, dist="normal", Ms=[1]),
    "llama7b_layer_3b_g128": dict(
        desc="Llama-7B-shaped decoder layer (qkv 4096->12288, o 4096->4096, gate/up "
             "4096->22016, down 11008->4096), 3-bit, group 128, M=1,4,16",
        linears=LLAMA7B_LAYER, bits=3, group=128, dist="normal", Ms=[1, 4, 16]),
    "opt175b_fc_2b_rowwise": dict(
        desc="OPT-175B-shaped FC1 12288->49152 and FC2 49152->12288, per-row, 2-bit, "
             "W~0.02*t(4), M=1",
        linears=[("fc1", 49152, 12288), ("fc2", 12288, 49152)], bits=2, group=0,
        dist="t4", Ms=[1]),
    "opt175b_fc_8b_rowwise": dict(
        desc="OPT-175B-shaped FC1 12288->49152 and FC2 49152->12288, per-row, 8-bit, "
             "W~0.02*t(4), M=1",
        linears=[("fc1", 49152, 12288), ("fc2", 12288, 49152)], bits=8, group=0,
        dist="t4", Ms=[1]),
    "llama13b_prefill_4b_g128": dict(
        desc="Llama-13B-shaped prefill GEMMs 5120->13824 and 13824->5120, 4-bit, "
             "group 128, x [2048, K]",
        linears=[("up", 13824, 5120), ("down", 5120, 13824)], bits=4, group=128,
        dist="normal", Ms=[2048]),
    "llama7b_stack32_4b_g128": dict(
        desc="32-layer 7B-shaped linear stack (q,k,v,o,gate,up,down per layer), 4-bit, "
             "group 128, ~3.5 GB packed, M=1,4,16,64",
        linears=[(f"L{l}.{nm}", n, k) for l in range(32) for (nm, n, k) in LLAMA7B_STACK_LAYER],
        bits=4, group=128, dist="normal", Ms=[1, 4, 16, 64]),
}
