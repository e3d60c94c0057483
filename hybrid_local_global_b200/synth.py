"""Seeded synthetic inputs. Holds none of the attention arithmetic.

Both the CUDA path and the CPU oracle read the tensors made here: tests
draw them (on the CPU or on the device), hand the very same bf16 values to
the kernels and, as uint16 bit patterns, to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, gen: torch.Generator, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """bf16 ~ N(0, scale^2), drawn in fp32 from `gen` then rounded."""
    x = torch.randn(tuple(shape), generator=gen, device=torch.device(device), dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def fill_randn_bf16_(t: torch.Tensor, gen: torch.Generator, scale: float = 1.0) -> torch.Tensor:
    """In-place bf16 ~ N(0, scale^2) fill, one leading slice at a time (no
    full-size fp32 temporary for multi-GiB caches)."""
    for i in range(t.shape[0]):
        x = torch.randn(tuple(t.shape[1:]), generator=gen, device=t.device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        t[i].copy_(x)
    return t


def fill_int8_cache_(cache, gen: torch.Generator):
    """Synthetic int8 cache rows: codes uniform on 0..255 and (min, step)
    near those of a N(0, 1) row of a few hundred channels (min about -3,
    step about 6 / 255), drawn from `gen` one leading slice at a time."""
    codes, params = cache.codes, cache.params
    for i in range(codes.shape[0]):
        c = torch.randint(0, 256, tuple(codes.shape[1:]), generator=gen, device=codes.device, dtype=torch.int32)
        codes[i].copy_(c)
        n = torch.randn(tuple(params.shape[1:]), generator=gen, device=params.device, dtype=torch.float32)
        params[i, ..., 0].copy_(-3.0 + 0.2 * n[..., 0])
        params[i, ..., 1].copy_((6.0 / 255.0) * (1.0 + 0.05 * n[..., 1]))
    return cache


def fill_cache_(cache, gen: torch.Generator):
    """A layer's cache buffer filled with synthetic rows: bf16 N(0, 1), or
    int8 rows (fill_int8_cache_) for an int8 cache object."""
    if isinstance(cache, torch.Tensor):
        return fill_randn_bf16_(cache, gen)
    return fill_int8_cache_(cache, gen)


def decode_lengths(batch: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Per-sequence KV lengths uniform on [lo, hi] (int32, CPU)."""
    g = generator(seed)
    return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (a copy on the host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
