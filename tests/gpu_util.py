"""Helpers shared by the GPU parity tests (no arithmetic of the method here:
inputs come from hybrid_local_global_b200.synth, expected values from the
oracle)."""
from __future__ import annotations

import numpy as np
import torch

from hybrid_local_global_b200 import synth

# Parity tolerance for bf16 outputs against the fp64 oracle.
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


def bf16_ulp(x: torch.Tensor) -> torch.Tensor:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = x.float().abs().clamp_min(2.0 ** -126)
    return torch.exp2(torch.floor(torch.log2(a)) - 7)


def assert_rotated_bf16(got: torch.Tensor, exp: torch.Tensor, x: torch.Tensor, what=""):
    """Rotated bf16 K against the bf16-rounded fp64 rotation. The kernel rounds
    its fp32 rotation to nearest, the reference rounds the exact value, so the
    two differ by at most one bf16 ulp where the values straddle a rounding
    boundary; the fp32 rotation (x0*c - x1*s with c, s of an fp32-rounded
    reduced angle) adds about 2^-22 * (|x0| + |x1|), bounded here by 2^-20."""
    xf = x.float()
    pair = xf.view(-1, 2).abs().sum(dim=1).repeat_interleave(2)
    tol = bf16_ulp(exp) + 2 ** -20 * pair
    d = (got.float() - exp.float()).abs()
    assert bool((d <= tol).all()), "%s: max excess %.3e" % (what, float((d - tol).max()))


# The prefill kernels take queries rotated and pre-multiplied by the logit
# scale in log2 units (scale * log2 e, an fp32 constant), rounded to bf16 once;
# decode rounds the rotated query itself. Keys are rotated and rounded to bf16
# by both.
LOG2E = 1.4426950408889634


def prefill_query_multiplier(scale: float) -> float:
    """The fp32 constant the prefill path multiplies rotated queries by."""
    return float(np.float32(np.float64(np.float32(scale)) * LOG2E))


def rotate_round(oracle, x: "torch.Tensor", pos, frac, theta, mult=1.0):
    """bf16 rows [B, S, H, D] -> the oracle's (p-)RoPE of row (b, s, h) at
    position pos[b] + s, times `mult`, rounded to bf16: the operands as the
    GPU path rounds them."""
    import torch
    B, S, H, D = x.shape
    xb = to_bits(x)
    y = np.empty((B, S, H, D), dtype=np.float64)
    for b in range(B):
        for s_ in range(S):
            for h in range(H):
                y[b, s_, h] = oracle.rope_bf16(xb[b, s_, h], int(pos[b]) + s_, frac, theta)
    return torch.from_numpy(y * mult).to(torch.bfloat16)


# bf16 unit roundoff (8 significant bits, round to nearest)
BF16_U = 2.0 ** -8


def rounding_bound(model: np.ndarray, v_absmax: float) -> float:
    """Largest |gpu - model| that the GPU's own bf16 roundings allow, the
    operands rounded as in `model`: every weight p_j is rounded to bf16
    (relative error <= u) and normalised by the sum of the unrounded
    weights, which moves an output by at most u * sum_j w_j |v_j| <=
    u * max|v|; the output itself is rounded to bf16 (<= u * |o|). A slack
    of 2^-10 covers the fp32 accumulations and the exp2 approximation."""
    return BF16_U * (v_absmax + float(np.abs(model).max())) + 2.0 ** -10


def assert_close_to_model(gpu, model, exact, v_absmax, what=""):
    """GPU output against the exact attention of its rounded operands within
    the rounding bound above (mean-abs within the parity tolerance 2e-3), and
    against the exact oracle within the model's own error plus that bound
    (the triangle inequality)."""
    tol = rounding_bound(model, v_absmax)
    assert_close(gpu, model, tol, MEAN_ABS, what="%s vs rounded-operand model" % what)
    e = np.abs(model - exact)
    assert_close(gpu, exact, float(e.max()) + tol, float(e.mean()) + MEAN_ABS, what="%s vs exact" % what)
