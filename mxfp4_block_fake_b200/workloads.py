"""Seeded synthetic workloads for MXFP4 block fake quantisation.

This module only draws inputs: shapes, value distributions, injected special
blocks and MoE group sizes. It holds none of the quantisation arithmetic, and
both the CUDA path's tests/bench and the CPU oracle's checks take their inputs
from here. Every draw uses a torch CPU Generator seeded per workload, so a
workload is the same bytes on every machine.

Workloads (all bf16 unless stated; sizes are the defaults, tests shrink them
with the same recipe):
  qat_linear_tiny  fp32 x [4,64], weight [32,64] ~ N(0,1), seed 0
  act_rowwise      [8192,4096] ~ N(0,1); 0.5% of the columns (20 of 4096,
                   drawn by the same generator) multiplied by 50, seed 1
  weight_dual      [14336,4096] ~ N(0, 0.02^2), seed 2
  train_step       x [16384,4096] = 0.5 * Student-t(4) (Z / sqrt(chi2_4 / 4)),
                   grad_out ~ N(0, (1e-3)^2), seed 3; injected: every 4096th
                   row-wise block of 32 all-zero, one block of bf16 subnormals
                   (amax 2^-130, row 3 block 1), and +inf / -inf / NaN blocks
                   (row 7, blocks 3 / 4 / 5)
  moe_grouped      [65536,7168] ~ N(0,1), seed 4; 256 group sizes drawn as a
                   multinomial of the rows over p ~ u^4, u ~ U(0,1); groups
                   0, 100 and 255 emptied into groups 1, 101 and 254
"""
from __future__ import annotations

import torch

SUBNORMAL_2_M130 = 0x0008  # bf16 bits of 2^-130 (8 * 2^-133)


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed)


def qat_linear_tiny(seed: int = 0):
    g = _gen(seed)
    x = torch.randn(4, 64, generator=g, dtype=torch.float32)
    w = torch.randn(32, 64, generator=g, dtype=torch.float32)
    return x, w


def act_rowwise(rows: int = 8192, cols: int = 4096, seed: int = 1, outlier_frac: float = 0.005,
                outlier_gain: float = 50.0) -> torch.Tensor:
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    n_out = max(1, round(outlier_frac * cols))
    cols_out = torch.randperm(cols, generator=g)[:n_out]
    x[:, cols_out] *= outlier_gain
    return x.to(torch.bfloat16)


def weight_dual(rows: int = 14336, cols: int = 4096, seed: int = 2, sigma: float = 0.02) -> torch.Tensor:
    g = _gen(seed)
    return (torch.randn(rows, cols, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)


def train_step(rows: int = 16384, cols: int = 4096, seed: int = 3, block: int = 32):
    """Returns (x, grad_out), both bf16 [rows, cols]."""
    g = _gen(seed)
    z = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    chi2 = torch.zeros(rows, cols, dtype=torch.float32)
    for _ in range(4):
        chi2 += torch.randn(rows, cols, generator=g, dtype=torch.float32).square()
    x = 0.5 * z / torch.sqrt(chi2 / 4.0)
    grad = torch.randn(rows, cols, generator=g, dtype=torch.float32) * 1e-3
    xb = x.to(torch.bfloat16)
    nb = cols // block
    # every 4096th row-wise block (row-major block numbering) all zero
    flat = xb.view(rows, nb * block)[:, : nb * block].reshape(-1, block) if cols % block == 0 else None
    if flat is not None:
        flat[::4096] = 0
    bits = xb.view(torch.int16)
    if rows > 3 and nb > 1:
        # one block of bf16 subnormals, magnitudes k * 2^-133 (k = 1..8), amax 2^-130
        mags = torch.randint(1, 9, (block,), generator=g, dtype=torch.int16)
        sgn = torch.randint(0, 2, (block,), generator=g, dtype=torch.int16) * -32768
        blk = mags | sgn
        blk[0] = SUBNORMAL_2_M130
        bits[3, block: 2 * block] = blk
    if rows > 7 and nb > 5:
        xb[7, 3 * block + 5] = float("inf")
        xb[7, 4 * block + 9] = float("-inf")
        xb[7, 5 * block + 17] = float("nan")
    return xb, grad.to(torch.bfloat16)


def train_step_grad(rows: int, cols: int, seed: int = 5, sigma: float = 1e-3) -> torch.Tensor:
    """Incoming gradient of the training-step workloads: bf16 ~ N(0, sigma^2)."""
    g = _gen(seed)
    return (torch.randn(rows, cols, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)


def moe_group_counts(rows: int, groups: int = 256, seed: int = 4, empty=(0, 100, 255)):
    """Multinomial group sizes over p ~ u^4; the listed groups are emptied into
    their neighbours (0 -> 1, 100 -> 101, 255 -> 254)."""
    g = _gen(seed + 1000)
    u = torch.rand(groups, generator=g, dtype=torch.float64)
    p = u ** 4
    draws = torch.multinomial(p, rows, replacement=True, generator=g)
    counts = torch.bincount(draws, minlength=groups).to(torch.int64)
    for e in empty:
        if e >= groups:
            continue
        to = e + 1 if e + 1 < groups and e + 1 not in empty else e - 1
        counts[to] += counts[e]
        counts[e] = 0
    return counts


def moe_grouped(rows: int = 65536, cols: int = 7168, groups: int = 256, seed: int = 4):
    """Returns (x bf16 [rows, cols], counts int64 [groups], offsets int64 [groups])."""
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32).to(torch.bfloat16)
    counts = moe_group_counts(rows, groups, seed)
    return x, counts, torch.cumsum(counts, 0)


def mixed(rows: int, cols: int, dtype=torch.bfloat16, seed: int = 9, specials: bool = True) -> torch.Tensor:
    """Parity-test input mixing every regime a block can be in: N(0,1) rows
    scaled by 2^U(-40, 40), a few x50 outlier columns, exact codebook values
    and midpoints times a power of two, all-zero and -0 blocks, bf16/fp32
    subnormals, and (with specials) scattered +inf, -inf and NaN."""
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    x *= torch.exp2(torch.randint(-40, 41, (rows, 1), generator=g).float())
    if cols >= 8:
        x[:, torch.randperm(cols, generator=g)[: max(1, cols // 200)]] *= 50
    n = rows * cols
    flat = x.view(-1)
    grid = torch.tensor([0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0, 7.0])
    idx = torch.randint(0, n, (n // 16,), generator=g)
    pick = grid[torch.randint(0, len(grid), (idx.numel(),), generator=g)]
    sgn = torch.where(torch.rand(idx.numel(), generator=g) < 0.5, -1.0, 1.0)
    flat[idx] = sgn * pick * torch.exp2(torch.randint(-10, 11, (idx.numel(),), generator=g).float())
    idx = torch.randint(0, n, (n // 64,), generator=g)
    flat[idx] = torch.where(torch.rand(idx.numel(), generator=g) < 0.5, 0.0, -0.0)
    if rows >= 4 and cols >= 64:
        r0 = int(torch.randint(0, rows - 3, (1,), generator=g))
        x[r0: r0 + 3, 0:64] = 0.0
        x[r0 + 1, 3] = -0.0
    tiny = 2.0 ** -133 if dtype == torch.bfloat16 else 2.0 ** -149
    idx = torch.randint(0, n, (n // 128,), generator=g)
    flat[idx] = torch.randint(-16, 17, (idx.numel(),), generator=g).float() * tiny
    if rows >= 2 and cols >= 64:
        r1 = int(torch.randint(0, rows, (1,), generator=g))
        x[r1, 32:64] = torch.randint(-127, 128, (32,), generator=g).float() * tiny
    if specials:
        for v in (float("inf"), float("-inf"), float("nan")):
            idx = torch.randint(0, n, (max(1, n // 20000),), generator=g)
            flat[idx] = v
    return x.to(dtype)


WORKLOADS = {
    "qat_linear_tiny": qat_linear_tiny,
    "act_rowwise": act_rowwise,
    "weight_dual": weight_dual,
    "train_step": train_step,
    "moe_grouped": moe_grouped,
}
