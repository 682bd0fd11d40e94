"""Seeded synthetic inputs for the NVFP4 quantize + GEMM workloads.

This module is shared by the tests, the benchmark and the smoke check. It holds no
arithmetic of the method (no scaling, rounding, encoding or layout): it only draws
random numbers with a seeded CPU generator and casts them to the input dtype. Both the
oracle and the CUDA path read the bytes it returns.

Workloads (shapes and distributions of the five synthetic configurations):
  tiny      A bf16 [16,512] ~ N(0,1), W bf16 [256,512] ~ N(0,0.02)
  per_token X bf16 [8192,7168] ~ N(0,1), 0.1% of entries (seeded randperm) scaled x50
  swiglu    X bf16 [4096, 2*14336] ~ N(0,1) (gate | up halves)
  decode    W bf16 [28672,8192] ~ N(0,0.02); A bf16 [M,8192] ~ N(0,1), M in {1,8,32}
  prefill   A bf16 [8192,8192] ~ N(0,1), W bf16 [8192,8192] ~ N(0,0.02)
"""
from __future__ import annotations

import numpy as np
import torch

SEEDS = {"tiny": 0, "per_token": 1, "swiglu": 2, "decode": 3, "prefill": 4}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float = 1.0, seed: int = 0, dtype=torch.bfloat16) -> torch.Tensor:
    """Seeded N(0, std^2) on the CPU, drawn in fp32 and cast once to `dtype`."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def with_outliers(shape, frac: float = 0.001, factor: float = 50.0, seed: int = 0,
                  dtype=torch.bfloat16) -> torch.Tensor:
    """N(0,1) with round(frac * numel) entries, picked by a seeded randperm, times `factor`."""
    g = _gen(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    n = x.numel()
    count = int(round(frac * n))
    idx = torch.randperm(n, generator=g)[:count]
    x.view(-1)[idx] *= factor
    return x.to(dtype)


def tiny(seed: int = SEEDS["tiny"]):
    a = normal((16, 512), 1.0, seed)
    w = normal((256, 512), 0.02, seed + 100)
    return a, w


def per_token(M: int = 8192, K: int = 7168, seed: int = SEEDS["per_token"]):
    return with_outliers((M, K), 0.001, 50.0, seed)


def swiglu(M: int = 4096, H: int = 14336, seed: int = SEEDS["swiglu"]):
    return normal((M, 2 * H), 1.0, seed)


def decode(M: int, N: int = 28672, K: int = 8192, seed: int = SEEDS["decode"]):
    w = normal((N, K), 0.02, seed)
    a = normal((M, K), 1.0, seed + 1000 + M)
    return a, w


def prefill(M: int = 8192, N: int = 8192, K: int = 8192, seed: int = SEEDS["prefill"]):
    a = normal((M, K), 1.0, seed)
    w = normal((N, K), 0.02, seed + 100)
    return a, w


def random_bytes(shape, seed: int, low: int = 0, high: int = 256) -> np.ndarray:
    """Seeded uniform integers in [low, high) as uint8 (raw packed operands / scale codes)."""
    g = _gen(seed)
    return torch.randint(low, high, tuple(shape), generator=g, dtype=torch.int32).to(torch.uint8).numpy()


def bits16(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16/fp16 CPU tensor as np.uint16 (no conversion)."""
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
