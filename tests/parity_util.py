"""Shared helpers of the parity tests: row sampling and the comparison bar.

Tolerances (fp32 accumulation of bf16 inputs, bf16 probabilities and bf16
output, against the fp64 oracle): O max-abs 2e-2 and mean-abs 2e-3, LSE
abs 1e-3; tables bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def sample_rows(wl, n_random: int = 512, seed: int = 0) -> np.ndarray:
    """Flat row ids (b*H_q + h)*C + r: for every (b, g) all rows of the first
    and the last Q-block of the group's first head (every tile boundary and the
    diagonal blocks), plus ``n_random`` uniform rows."""
    rows = []
    G = wl.group
    for b in range(wl.B):
        for g in range(wl.H_kv):
            h = g * G
            base = (b * wl.H_q + h) * wl.C
            first = np.arange(0, min(wl.blk, wl.C))
            last = np.arange(max(0, wl.C - wl.blk), wl.C)
            rows.append(base + first)
            rows.append(base + last)
    rng = np.random.default_rng(seed)
    rows.append(rng.integers(0, wl.B * wl.H_q * wl.C, size=n_random))
    return np.unique(np.concatenate(rows).astype(np.int64))


def compare(O_gpu: torch.Tensor, LSE_gpu: torch.Tensor, O_ref: np.ndarray, LSE_ref: np.ndarray,
            rows=None, o_max=O_MAX_ABS, o_mean=O_MEAN_ABS, lse_abs=LSE_ABS):
    D = O_gpu.shape[-1]
    O = O_gpu.float().cpu().numpy().reshape(-1, D)
    L = LSE_gpu.float().cpu().numpy().reshape(-1)
    if rows is not None:
        O, L = O[rows], L[rows]
    O_ref = O_ref.reshape(-1, D)
    L_ref = LSE_ref.reshape(-1)
    assert np.isfinite(O).all(), "non-finite values in O"
    err = np.abs(O - O_ref)
    assert err.max() <= o_max, f"O max-abs {err.max():.3e} > {o_max}"
    assert err.mean() <= o_mean, f"O mean-abs {err.mean():.3e} > {o_mean}"
    inf_ref = np.isneginf(L_ref)
    assert np.array_equal(np.isneginf(L), inf_ref), "LSE -inf pattern differs"
    if (~inf_ref).any():
        lerr = np.abs(L[~inf_ref] - L_ref[~inf_ref])
        assert lerr.max() <= lse_abs, f"LSE abs {lerr.max():.3e} > {lse_abs}"
    return float(err.max()), float(err.mean())
