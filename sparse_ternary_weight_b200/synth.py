"""Seeded synthetic inputs (weights and activations) for tests and benchmarks.

This module holds no arithmetic of the quantisation method: it only draws
random numbers and rounds activations to bf16 storage.  Both the CUDA path and
the CPU oracle receive their inputs from here, and nothing else is shared.

Workloads (shapes borrowed from LLaMA-3.2; no real weights or data are used):

* tiny: one linear N=64, K=256, W ~ N(0, 0.02^2), X ~ N(0,1) bf16, seed 0.
* 1B decode: 16 layers of q/o 2048x2048, k/v 512x2048, gate/up 8192x2048,
  down 2048x8192; W ~ N(0, 0.02^2) with 1% of entries multiplied by 8.
* 3B: 28 layers of q/o 3072x3072, k/v 1024x3072, gate/up 8192x3072,
  down 3072x8192; W ~ Student-t(4) scaled to std 0.02 (t(4) has variance 2).

Seeds: weight seed = 1000*cfg + 16*layer + proj (proj q,k,v,o,gate,up,down =
0..6); activation seed = weight seed + 500000.  NumPy PCG64 streams.  A
device-side variant (torch Philox, same distributions, different streams) is
offered for benchmarks whose full weight sets would take minutes to draw on
the host; parity never uses it.
"""
from __future__ import annotations

import numpy as np

PROJ = ("q", "k", "v", "o", "gate", "up", "down")

STACKS = {
    # name: (cfg index, layers, {proj: (N, K)})
    "1b": (2, 16, {"q": (2048, 2048), "k": (512, 2048), "v": (512, 2048), "o": (2048, 2048),
                   "gate": (8192, 2048), "up": (8192, 2048), "down": (2048, 8192)}),
    "3b": (3, 28, {"q": (3072, 3072), "k": (1024, 3072), "v": (1024, 3072), "o": (3072, 3072),
                   "gate": (8192, 3072), "up": (8192, 3072), "down": (3072, 8192)}),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def weight_seed(cfg: int, layer: int, proj: str) -> int:
    return 1000 * cfg + 16 * layer + PROJ.index(proj)


def act_seed(cfg: int, layer: int, proj: str) -> int:
    return weight_seed(cfg, layer, proj) + 500000


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) and return the uint16 bits."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def weights_normal(N: int, K: int, seed: int, std: float = 0.02,
                   outlier_frac: float = 0.0, outlier_mult: float = 8.0) -> np.ndarray:
    g = rng(seed)
    W = g.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    if outlier_frac > 0:
        m = g.random((N, K), dtype=np.float32) < outlier_frac
        W[m] *= np.float32(outlier_mult)
    return W


def weights_student_t(N: int, K: int, seed: int, df: float = 4.0, std: float = 0.02) -> np.ndarray:
    g = rng(seed)
    scale = std / np.sqrt(df / (df - 2.0))
    return (g.standard_t(df, size=(N, K)) * scale).astype(np.float32)


def activations_bf16(M: int, K: int, seed: int) -> np.ndarray:
    """X ~ N(0,1) rounded to bf16; returned as uint16 bits [M,K]."""
    return f32_to_bf16_bits(rng(seed).standard_normal((M, K), dtype=np.float32))


def stack_weight(stack: str, layer: int, proj: str) -> np.ndarray:
    cfg, _, shapes = STACKS[stack]
    N, K = shapes[proj]
    s = weight_seed(cfg, layer, proj)
    if stack == "1b":
        return weights_normal(N, K, s, 0.02, outlier_frac=0.01, outlier_mult=8.0)
    return weights_student_t(N, K, s)


def stack_activations(stack: str, layer: int, proj: str, M: int) -> np.ndarray:
    cfg, _, shapes = STACKS[stack]
    _, K = shapes[proj]
    return activations_bf16(M, K, act_seed(cfg, layer, proj))


def tiny():
    """The tiny single-linear case: (W f32 [64,256], X bf16 bits [1,256])."""
    return weights_normal(64, 256, 0, 0.02), activations_bf16(1, 256, 500000)


# ---- device-side draws for benchmarks (torch; same distributions) ----

def torch_stack_weight(stack: str, layer: int, proj: str, device="cuda"):
    import torch
    cfg, _, shapes = STACKS[stack]
    N, K = shapes[proj]
    g = torch.Generator(device=device)
    g.manual_seed(weight_seed(cfg, layer, proj))
    if stack == "1b":
        W = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02
        m = torch.rand((N, K), generator=g, device=device) < 0.01
        return torch.where(m, W * 8.0, W)
    # Student-t(4) = Z / sqrt(V/4), V ~ chi^2(4) = sum of 4 squared normals
    z = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    v = torch.zeros_like(z)
    for _ in range(4):
        e = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
        v.add_(e * e)
    t = z / torch.sqrt(v / 4.0)
    return t * (0.02 / np.sqrt(2.0))


def torch_activations_bf16(M: int, K: int, seed: int, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn((M, K), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
