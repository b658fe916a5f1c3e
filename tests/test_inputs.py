"""The seeded generators are deterministic and row subsets match the full draw."""
import numpy as np
import torch

import wq_inputs


def test_weight_rows_subset_matches_full():
    full = wq_inputs.weight_f16(0, 3, 600, 64, dist="t4")
    rows = np.array([599, 0, 257, 256, 12])
    part = wq_inputs.weight_f16(0, 3, 600, 64, dist="t4", rows=rows)
    assert np.array_equal(full[rows].view(np.uint16), part.view(np.uint16))
    again = wq_inputs.weight_f16(0, 3, 600, 64, dist="t4")
    assert np.array_equal(full.view(np.uint16), again.view(np.uint16))
    assert full.dtype == np.float16 and np.all(np.isfinite(full))


def test_weight_distribution_shape():
    w = wq_inputs.weight_f16(0, 1, 512, 512).astype(np.float64)
    assert abs(w.std() - 0.02) < 1e-3 and abs(w.mean()) < 1e-3


def test_activations_bf16():
    x = wq_inputs.activations_bf16(0, 2, 3, 4096)
    assert x.dtype == torch.bfloat16 and x.shape == (3, 4096)
    assert torch.equal(x, wq_inputs.activations_bf16(0, 2, 3, 4096))
    assert abs(x.float().std().item() - 1.0) < 0.05
