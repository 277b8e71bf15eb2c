"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method: it only draws random numbers.
Weights are fp32 ~ N(0, 0.02^2) (0.02 read as the standard deviation) and
activations are bf16 ~ N(0, 1), drawn from a torch.Generator seeded per tensor.
A 27B-shaped decoder layer has four products (hidden 5120, FFN 17408):
fused QKV 5120->7168, O 5120->5120, gate+up 5120->34816 and down 17408->5120.
"""
from __future__ import annotations

import torch

HIDDEN, FFN = 5120, 17408
# (name, K = input features, N = output features)
LAYER_SHAPES = (("qkv", HIDDEN, 7168), ("o", HIDDEN, HIDDEN), ("gate_up", HIDDEN, 2 * FFN),
                ("down", FFN, HIDDEN))
N_LAYERS = 64
WEIGHT_STD = 0.02


def seed_of(base: int, layer: int, matrix: int) -> int:
    """Seed of matrix `matrix` (0..3) of layer `layer`: base + 4*layer + matrix."""
    return int(base) + 4 * int(layer) + int(matrix)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 [N][K] ~ N(0, 0.02^2)."""
    w = torch.randn((N, K), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return w.mul_(WEIGHT_STD)


def activations(M: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [M][K] ~ N(0, 1) (drawn in fp32, then rounded to bf16)."""
    x = torch.randn((M, K), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
