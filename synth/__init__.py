"""Seeded synthetic inputs for the quantization workloads.

This module is shared by the tests, the benchmark and the smoke check.  It
draws random bf16 tensors and integer splits and holds none of the
quantization arithmetic.  Every generator is deterministic for a given seed
and device (the CPU and CUDA generators of torch give different streams, so a
test draws once and copies to the other side).

Workloads (shapes from the expert-prequantization, split-quantization and
fused-epilogue pages; the model weights themselves are not needed, only their
shapes and a plausible value distribution):

* tiny MXFP8 group: 4 experts [64, 256], N(0,1) * 2^U(-4,4) per row
* Qwen3-30B-A3B refit: 128 experts/layer, gate_up [1536, 2048] and down
  [2048, 768], N(0, 0.02), 48 layers, seed 2 + layer
* row-scaled NVFP4 split: [16384, 4096] N(0,1) with 1% outliers x20; rows
  split over 64 experts by multinomial(Dirichlet(0.3))
* fused residual + RMSNorm: x, r [T, 7168] N(0,1), gamma U(0.5, 1.5), eps 1e-6
* AllReduce epilogue: the fused workload's x as the sum of n rank partials,
  each N(0, 1/n) [T, 7168] (a row-parallel projection's partial outputs)
* Qwen3-235B-A22B prequant: 128 experts/layer, gate_up [3072, 4096] and down
  [4096, 1536], N(0, 0.02), 94 layers, seed 5 + layer

``moe_layer`` draws one projection of one layer of either MoE workload from
its seed (``layer_seed``), so a sweep can regenerate every layer in place.
"""
from __future__ import annotations

import numpy as np
import torch

QWEN3_30B = dict(layers=48, experts=128, gate_up=(1536, 2048), down=(2048, 768), std=0.02, seed=2)
QWEN3_235B = dict(layers=94, experts=128, gate_up=(3072, 4096), down=(4096, 1536), std=0.02, seed=5)
SPLIT_ACT = dict(tokens=16384, hidden=4096, experts=64, alpha=0.3, outlier_p=0.01, outlier_mul=20.0, seed=3)
FUSED_NORM = dict(hidden=7168, eps=1e-6, seed=4, tokens=tuple(2 ** i for i in range(13)))
TINY = dict(experts=4, shape=(64, 256), seed=1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float = 1.0, seed: int = 0, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and rounded to bf16 by torch."""
    g = _gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def tiny_group(seed: int = TINY["seed"], experts: int = TINY["experts"], shape=TINY["shape"], device="cpu"):
    """Experts of N(0,1) rows, each row times 2^u with u ~ U(-4, 4)."""
    g = _gen(seed, device)
    out = []
    for _ in range(experts):
        x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
        u = torch.rand(shape[0], 1, generator=g, device=device, dtype=torch.float32) * 8.0 - 4.0
        out.append((x * torch.exp2(u)).to(torch.bfloat16))
    return out


def expert_stack(n: int, shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """n same-shape expert matrices stacked as one [n, rows, cols] bf16 tensor."""
    return normal_bf16((n, *shape), std=std, seed=seed, device=device)


def layer_seed(cfg: dict, layer: int, proj: str, rank: int = 0) -> int:
    """Seed of one projection of one MoE layer: the workload's seed + layer
    (+500 for the down projection, +1000 per rank of a multi-GPU run)."""
    return int(cfg["seed"]) + int(layer) + 1000 * int(rank) + (0 if proj == "gate_up" else 500)


def moe_layer(cfg: dict, layer: int, proj: str, device="cuda", rank: int = 0, out=None) -> torch.Tensor:
    """The experts of one projection ("gate_up" or "down") of layer ``layer``
    as one [experts, rows, cols] bf16 tensor, N(0, std^2), regenerated from
    its seed alone.  Drawn in place (each value rounded once to bf16), so a
    layer of the largest workload needs no temporary beyond its own 3.2 GB."""
    shape = (cfg["experts"], *cfg[proj])
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    assert tuple(out.shape) == shape and out.dtype == torch.bfloat16
    out.normal_(0.0, float(cfg["std"]), generator=_gen(layer_seed(cfg, layer, proj, rank), out.device))
    return out


def split_activation(tokens=SPLIT_ACT["tokens"], hidden=SPLIT_ACT["hidden"], seed=SPLIT_ACT["seed"],
                     outlier_p=SPLIT_ACT["outlier_p"], outlier_mul=SPLIT_ACT["outlier_mul"], device="cpu"):
    """[tokens, hidden] N(0,1) bf16 with a Bernoulli(outlier_p) mask scaled by outlier_mul."""
    g = _gen(seed, device)
    x = torch.randn(tokens, hidden, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(tokens, hidden, generator=g, device=device, dtype=torch.float32) < outlier_p
    x = torch.where(mask, x * outlier_mul, x)
    return x.to(torch.bfloat16)


def dirichlet_splits(tokens=SPLIT_ACT["tokens"], experts=SPLIT_ACT["experts"], alpha=SPLIT_ACT["alpha"],
                     seed=SPLIT_ACT["seed"], force_empty=()):
    """Row counts per expert: multinomial(tokens, Dirichlet(alpha * 1)).

    ``force_empty`` lists experts whose rows are moved to their right
    neighbour (or left, for the last), to force empty splits."""
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.full(experts, alpha))
    counts = rng.multinomial(tokens, p).astype(np.int64)
    for e in force_empty:
        dst = e + 1 if e + 1 < experts else e - 1
        counts[dst] += counts[e]
        counts[e] = 0
    assert counts.sum() == tokens
    return counts


def fused_norm_inputs(tokens: int, hidden=FUSED_NORM["hidden"], seed=FUSED_NORM["seed"], device="cpu"):
    """x, residual ~ N(0,1) [tokens, hidden]; gamma ~ U(0.5, 1.5) [hidden]; all bf16."""
    g = _gen(seed, device)
    x = torch.randn(tokens, hidden, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    r = torch.randn(tokens, hidden, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    gamma = (torch.rand(hidden, generator=g, device=device, dtype=torch.float32) + 0.5).to(torch.bfloat16)
    return x, r, gamma


def rank_partials(ranks: int, tokens: int, hidden=FUSED_NORM["hidden"], seed=FUSED_NORM["seed"], device="cpu"):
    """``ranks`` partial inputs ~ N(0, 1/ranks) [tokens, hidden] of a tensor-parallel
    AllReduce (their sum is distributed like the fused workload's x), plus the
    residual ~ N(0,1) and gamma ~ U(0.5, 1.5); all bf16."""
    g = _gen(seed + 1000 * ranks, device)
    xs = [(torch.randn(tokens, hidden, generator=g, device=device, dtype=torch.float32) / ranks ** 0.5)
          .to(torch.bfloat16) for _ in range(ranks)]
    r = torch.randn(tokens, hidden, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    gamma = (torch.rand(hidden, generator=g, device=device, dtype=torch.float32) + 0.5).to(torch.bfloat16)
    return xs, r, gamma


def random_finite_bf16(shape, seed: int = 0, device="cpu") -> torch.Tensor:
    """Uniformly random finite bf16 bit patterns (all exponents, subnormals and
    both zeros included) -- a stress input covering every scale."""
    g = _gen(seed, device)
    bits = torch.randint(0, 1 << 16, shape, generator=g, device=device, dtype=torch.int32)
    exp = (bits >> 7) & 0xFF
    bits = torch.where(exp == 0xFF, bits & ~(0x1 << 7), bits)  # exponent 0xFF -> 0xFE
    return bits.to(torch.int16).view(torch.bfloat16)


def blockwise_scaled(shape, block: int, seed: int = 0, lo: float = -40.0, hi: float = 40.0,
                     zero_frac: float = 0.05, device="cpu") -> torch.Tensor:
    """N(0,1) values where each run of ``block`` consecutive row elements is
    scaled by its own 2^U(lo, hi); a fraction of blocks is all zero and a few
    elements are negative zero -- exercises every scale path."""
    g = _gen(seed, device)
    rows, cols = shape
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    nb = cols // block
    u = torch.rand(rows, nb, 1, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo
    z = torch.rand(rows, nb, 1, generator=g, device=device, dtype=torch.float32) < zero_frac
    x = x.view(rows, nb, block) * torch.exp2(u)
    x = torch.where(z, torch.zeros_like(x), x)
    x = x.view(rows, cols)
    nz = torch.rand(rows, cols, generator=g, device=device, dtype=torch.float32) < 0.002
    x = torch.where(nz, torch.full_like(x, -0.0), x)
    return x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """A CPU bf16 tensor as a numpy uint16 array (bit pattern, no copy of values)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def random_payload(rows: int, cols: int, fmt: int, seed: int = 0) -> np.ndarray:
    """Random quantized payload bytes: e4m3 codes [rows, cols] without the two
    NaN codes (fmt 0) or packed e2m1 pairs [rows, cols/2] (fmt 1)."""
    rng = np.random.default_rng(seed)
    if fmt == 0:
        q = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
        q[(q & 0x7F) == 0x7F] = 0x00
        return q
    return rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)


def random_scale_bytes(n: int, fmt: int, seed: int = 0) -> np.ndarray:
    """Random scale bytes: E8M0 0..254 (fmt 0) or finite non-negative e4m3
    codes 0..126 (fmt 1)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 255 if fmt == 0 else 127, size=n, dtype=np.uint8)


def random_amax(n: int, seed: int = 0, lo: float = -20.0, hi: float = 20.0) -> np.ndarray:
    """Random positive binary32 amax values spread over 2^lo .. 2^hi."""
    rng = np.random.default_rng(seed)
    return (np.exp2(rng.uniform(lo, hi, size=n)) * rng.uniform(1.0, 2.0, size=n)).astype(np.float32)


def merge_partials(splits: int, tokens: int, hidden: int, seed: int = 0):
    """Flash-decoding partial outputs float32 [S, T, H] (N(0,1) times a per
    split-and-token factor 2^U(-4,4)) and their log-sum-exps float32 [S, T]
    (U(-6, 6))."""
    rng = np.random.default_rng(seed)
    O = rng.standard_normal((splits, tokens, hidden)) * np.exp2(rng.uniform(-4, 4, (splits, tokens, 1)))
    lse = rng.uniform(-6, 6, (splits, tokens))
    return O.astype(np.float32), lse.astype(np.float32)
