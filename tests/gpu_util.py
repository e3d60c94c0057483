"""Helpers shared by the GPU parity tests (no arithmetic of the method here:
inputs come from hybrid_local_global_b200.synth, expected values from the
oracle)."""
from __future__ import annotations

import numpy as np
import torch

from hybrid_local_global_b200 import synth

# Spec tolerance for bf16 outputs against the fp64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_bits(t: torch.Tensor) -> np.ndarray:
    return synth.bits(t)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close(gpu: np.ndarray, ref: np.ndarray, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    err = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    assert np.isfinite(gpu).all(), "%s: non-finite GPU output" % what
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= max_abs and mean <= mean_abs, "%s: max abs %.3e (tol %.1e), mean abs %.3e (tol %.1e)" % (
        what, mx, max_abs, mean, mean_abs)
    return mx, mean


def sample_rows(B, Hq, S, n_random, seed, window=0, prior=0, extra_i=()):
    """Rows (b, h, i): first/last rows of every head, rows around the window
    boundary, and `n_random` seeded random rows."""
    rng = np.random.default_rng(seed)
    special = {0, 1, S - 1, S // 2} | set(i for i in extra_i if 0 <= i < S)
    if window:
        for c in (window - 1, window, window + 1, 2 * window - 1, 2 * window):
            if 0 <= c - prior < S:
                special.add(c - prior)
    rows = set()
    for b in range(B):
        for h in range(Hq):
            for i in special:
                if 0 <= i < S:
                    rows.add((b, h, i))
    for _ in range(n_random):
        rows.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(S))))
    return np.array(sorted(rows), dtype=np.int32)


def gather_rows(out: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """out [B,S,Hq,D] -> [R,D] for rows (b, h, i)."""
    idx_b = torch.as_tensor(rows[:, 0], device=out.device, dtype=torch.long)
    idx_h = torch.as_tensor(rows[:, 1], device=out.device, dtype=torch.long)
    idx_i = torch.as_tensor(rows[:, 2], device=out.device, dtype=torch.long)
    return out[idx_b, idx_i, idx_h].float().cpu().double().numpy()
