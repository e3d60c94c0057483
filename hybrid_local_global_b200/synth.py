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


def decode_lengths(batch: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Per-sequence KV lengths uniform on [lo, hi] (int32, CPU)."""
    g = generator(seed)
    return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (a copy on the host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
