"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_attention_fractal_b200 import synth

# Output tolerance for bf16 inputs with fp32 accumulation, against the fp64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 2e-3


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def small(name, B, T, H, W, heads, d, block, patch, thr, sta=None, alpha=1.5, seed=11, iid=False):
    return synth.Workload(name, B, T, H, W, heads, d, block, patch, thr, sta, alpha, seed, iid)


def lists_to_keep(kv_count: torch.Tensor, kv_idx: torch.Tensor, nb: int) -> np.ndarray:
    cnt = kv_count.cpu().numpy().reshape(-1)
    idx = kv_idx.cpu().numpy().reshape(-1, nb)
    keep = np.zeros((cnt.size, nb), dtype=bool)
    for r in range(cnt.size):
        row = idx[r, :cnt[r]]
        assert np.all(np.diff(row) > 0), "kv_idx rows must be strictly ascending"
        assert row.size == 0 or (row.min() >= 0 and row.max() < nb)
        keep[r, row] = True
    return keep.reshape(tuple(kv_count.shape) + (nb,))


def compare_outputs(got: np.ndarray, want: np.ndarray, rows_mask=None):
    """Max-abs and mean-abs error of bf16 outputs vs the oracle over the rows selected."""
    if rows_mask is not None:
        got = got[rows_mask]
        want = want[rows_mask]
    err = np.abs(got - want)
    return float(err.max()), float(err.mean())
