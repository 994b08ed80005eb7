"""Helpers shared by the parity tests: device tensors from the seeded
generator and the comparison rules (tolerances, near-tie rule for top-M)."""
from __future__ import annotations

import numpy as np
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa

# Output tolerances (max abs error): 1e-4 for fp32 workloads, 2e-2 for bf16.
TOL = {"f32": 1e-4, "bf16": 2e-2}
# Top-M: positions that differ from the oracle's set must sit within this
# relative gap of the oracle's M-th largest score.
TIE_REL = 1e-3


def torch_dtype(wl):
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def dev(x, dtype=None, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)


def check_topm(gpu_idx, gpu_cnt, ref_idx, ref_cnt, ref_scores):
    """Compare index sets row by row with the near-tie rule.

    gpu_idx/ref_idx: [rows, M]; ref_scores: [rows, L] (oracle, fp64)."""
    gpu_idx = np.asarray(gpu_idx)
    ref_idx = np.asarray(ref_idx)
    np.testing.assert_array_equal(np.asarray(gpu_cnt), np.asarray(ref_cnt))
    swaps = 0
    for r in range(ref_idx.shape[0]):
        c = int(ref_cnt[r])
        g = gpu_idx[r, :c]
        assert np.all(gpu_idx[r, c:] == -1), f"row {r}: padding"
        assert np.all(np.diff(g) > 0), f"row {r}: not ascending/unique"
        o = ref_idx[r, :c]
        if np.array_equal(g, o):
            continue
        sc = ref_scores[r]
        valid = sc[np.isfinite(sc)]
        tau = np.sort(valid)[::-1][c - 1]
        bound = TIE_REL * max(abs(tau), 1e-6 * valid.max())
        diff = np.setxor1d(g, o)
        assert np.all((diff >= 0) & (diff < sc.size)), f"row {r}: index out of range"
        gaps = np.abs(sc[diff] - tau)
        assert np.all(gaps <= bound), (
            f"row {r}: {diff.size} positions differ, worst gap {gaps.max():.3e} > {bound:.3e}")
        swaps += diff.size // 2
    return swaps


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0
