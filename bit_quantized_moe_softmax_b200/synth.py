"""Seeded synthetic inputs for the ds4 routed-MoE layer.

This module only draws random numbers and places them in buffers: it holds
none of the layer's arithmetic (no dequantization, routing, packing or FFN).
Both the CUDA path's tests and the CPU oracle read the tensors it returns.

Recipes (the pages publish no weights or prompts; these stand in for them):
  * x ~ N(0, 1); router rows ~ N(0, 0.02) (or N(0, 1/H) where the router
    logits themselves should be N(0, 1)); shared expert ~ N(0, 0.02) rounded
    to bfloat16.
  * quantized experts, small shapes: N(0, 0.02) float weights that each side
    packs with its own packer.
  * quantized experts, full shapes: the packed fields drawn directly -- every
    byte uniform, except the binary16 scales d (and dmin) which are uniform in
    [1e-3, 4e-3] (4-bit blocks: [1e-4, 4e-4], the range a packer gives
    N(0, 0.02) weights, since their codes and 6-bit scales reach 15 and 63).
  * grid: 256 distinct rows of 8 magnitudes drawn from {8, 25, 43}.
  * Zipf(s) expert popularity: router bias b_e = ln p_{pi(e)}, p_r ~ r^-s over
    ranks r = 1..E, pi a seeded permutation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

Q2_BYTES = 84
IQ2_BYTES = 66
Q4_BYTES = 144
QK = 256


# Scales of the chained-layer workload: superblock scales 8x below the
# single-layer interval and a shared expert of std 0.01, so that the routed and
# the shared part each add about 0.1 (std) to x ~ N(0, 1) per layer and 8
# residual steps stay O(1).
CHAIN_D_RANGE = (1e-3 / 8, 4e-3 / 8)
CHAIN_SHARED_STD = 0.01


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, g: torch.Generator, device="cpu") -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def bf16_normal(shape, std: float, g: torch.Generator, device="cpu") -> torch.Tensor:
    """N(0, std) drawn in float32, converted to bfloat16 by torch (round to nearest even)."""
    return normal(shape, std, g, device).to(torch.bfloat16)


def grid_table(seed: int = 0) -> torch.Tensor:
    """[256, 8] uint8: rows of magnitudes from {8, 25, 43}, pairwise distinct (redrawn on repeat)."""
    g = gen(seed)
    vals = torch.tensor([8, 25, 43], dtype=torch.uint8)
    rows, seen = [], set()
    while len(rows) < 256:
        r = vals[torch.randint(0, 3, (8,), generator=g)]
        key = tuple(r.tolist())
        if key in seen:
            continue
        seen.add(key)
        rows.append(r)
    return torch.stack(rows)


def _fp16_uniform(n: int, lo: float, hi: float, g, device) -> torch.Tensor:
    return (torch.rand(n, generator=g, device=device) * (hi - lo) + lo).to(torch.float16)


def random_q2k_blocks(n_blocks: int, g, device="cpu", lo=1e-3, hi=4e-3) -> torch.Tensor:
    """[n_blocks, 84] uint8 Q2_K-style blocks with uniform bytes and d, dmin ~ U[lo, hi] (binary16)."""
    b = torch.randint(0, 256, (n_blocks, Q2_BYTES), generator=g, device=device, dtype=torch.uint8)
    dd = _fp16_uniform(2 * n_blocks, lo, hi, g, device).view(torch.uint8).view(n_blocks, 4)
    b[:, 80:84] = dd
    return b


def random_q4k_blocks(n_blocks: int, g, device="cpu", lo=1e-4, hi=4e-4) -> torch.Tensor:
    """[n_blocks, 144] uint8 Q4_K-style blocks with uniform bytes and d, dmin ~ U[lo, hi] (binary16)."""
    b = torch.randint(0, 256, (n_blocks, Q4_BYTES), generator=g, device=device, dtype=torch.uint8)
    dd = _fp16_uniform(2 * n_blocks, lo, hi, g, device).view(torch.uint8).view(n_blocks, 4)
    b[:, 0:4] = dd
    return b


def random_iq2_blocks(n_blocks: int, g, device="cpu", lo=1e-3, hi=4e-3) -> torch.Tensor:
    """[n_blocks, 66] uint8 IQ2_XXS-style blocks with uniform bytes and d ~ U[lo, hi] (binary16)."""
    b = torch.randint(0, 256, (n_blocks, IQ2_BYTES), generator=g, device=device, dtype=torch.uint8)
    d = _fp16_uniform(n_blocks, lo, hi, g, device).view(torch.uint8).view(n_blocks, 2)
    b[:, 0:2] = d
    return b


def zipf_bias(E: int, s: float, seed: int) -> torch.Tensor:
    """Router bias b_e = ln p_{pi(e)} with p_r proportional to r^-s (r = 1..E)."""
    g = gen(seed)
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    perm = torch.randperm(E, generator=g)
    return torch.log(p[perm]).to(torch.float32)


@dataclass(frozen=True)
class Shape:
    H: int
    I: int
    E: int
    k: int
    shared: bool = True


TINY = Shape(H=256, I=128, E=8, k=2)
FULL = Shape(H=4096, I=2048, E=256, k=8)


def float_layer(shape: Shape, seed: int, router_std=0.02, expert_std=0.02, shared_std=0.02,
                bias: torch.Tensor | None = None, device="cpu") -> dict:
    """A layer with float expert weights (to be packed by each side's packer).

    Keys: W_r [E,H] f32, b_r [E] f32 or None, grid [256,8] u8,
    gate_f/up_f [E,I,H] f32, down_f [E,H,I] f32, sh_gate/sh_up [I,H] bf16, sh_down [H,I] bf16.
    """
    g = gen(seed, device)
    H, I, E = shape.H, shape.I, shape.E
    layer = dict(H=H, I=I, E=E, k=shape.k)
    layer["W_r"] = normal((E, H), router_std, g, device)
    layer["b_r"] = bias
    layer["grid"] = grid_table(seed)
    layer["gate_f"] = normal((E, I, H), expert_std, g, device)
    layer["up_f"] = normal((E, I, H), expert_std, g, device)
    layer["down_f"] = normal((E, H, I), expert_std, g, device)
    if shape.shared:
        layer["sh_gate"] = bf16_normal((I, H), shared_std, g, device)
        layer["sh_up"] = bf16_normal((I, H), shared_std, g, device)
        layer["sh_down"] = bf16_normal((H, I), shared_std, g, device)
    return layer


def packed_layer(shape: Shape, seed: int, router_std=0.02, shared_std=0.02,
                 bias: torch.Tensor | None = None, device="cpu", d_range=None, expert_bits=2) -> dict:
    """A layer whose quantized experts are drawn directly as packed blocks.

    Keys: W_r, b_r, grid as in float_layer; gate/up [E, I*H/256, 66] u8,
    down [E, H*I/256, 84] u8 (expert_bits 4: all three [E, n/256, 144] u8,
    and expert_bits = 4); sh_gate/sh_up/sh_down bf16.  d_range: the interval
    of the binary16 superblock scales d (and dmin); default [1e-3, 4e-3]
    ([1e-4, 4e-4] for 4-bit blocks).
    """
    g = gen(seed, device)
    H, I, E = shape.H, shape.I, shape.E
    nb = I * H // QK
    layer = dict(H=H, I=I, E=E, k=shape.k)
    layer["W_r"] = normal((E, H), router_std, g, device)
    layer["b_r"] = bias
    layer["grid"] = grid_table(seed)
    if expert_bits == 4:
        lo, hi = d_range or (1e-4, 4e-4)
        for name in ("gate", "up", "down"):
            layer[name] = random_q4k_blocks(E * nb, g, device, lo, hi).view(E, nb, Q4_BYTES)
        layer["expert_bits"] = 4
    else:
        lo, hi = d_range or (1e-3, 4e-3)
        layer["gate"] = random_iq2_blocks(E * nb, g, device, lo, hi).view(E, nb, IQ2_BYTES)
        layer["up"] = random_iq2_blocks(E * nb, g, device, lo, hi).view(E, nb, IQ2_BYTES)
        layer["down"] = random_q2k_blocks(E * nb, g, device, lo, hi).view(E, nb, Q2_BYTES)
    if shape.shared:
        layer["sh_gate"] = bf16_normal((I, H), shared_std, g, device)
        layer["sh_up"] = bf16_normal((I, H), shared_std, g, device)
        layer["sh_down"] = bf16_normal((H, I), shared_std, g, device)
    return layer


def tokens(n: int, H: int, seed: int, dtype=torch.float32, device="cpu") -> torch.Tensor:
    """x ~ N(0, 1), [n, H]; bfloat16 activations are the float32 draws rounded by torch."""
    g = gen(seed, device)
    return normal((n, H), 1.0, g, device).to(dtype)


def router_std_unit_logits(H: int) -> float:
    """Router row std that makes x . w ~ N(0, 1) for x ~ N(0, 1)."""
    return 1.0 / math.sqrt(H)
