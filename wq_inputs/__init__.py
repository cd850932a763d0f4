"""Seeded synthetic inputs shared by the CUDA path's tests, the oracle's tests and the benchmark.

This module only draws random numbers and lays them out; it holds none of
the quantisation or matmul arithmetic.  Every generator takes an explicit
seed and uses its own ``torch.Generator``, so the same call always yields the
same bytes.  Weights are drawn in binary32 and, where a workload says bf16,
rounded to bf16 by torch (round to nearest even); the rounded bytes are what
both the CUDA path and the oracle receive.

Workload shapes (weights stored [N][K], one row per output channel, K the
reduction axis):
  tiny        K=256, N=512, binary32 weights ~ N(0, 0.02) with 4 entries set to
              +-1.0; one bf16 activation vector ~ N(0, 1).
  decode_up   K=4096, N=14336 (an LLM MLP up-projection), bf16 weights
              ~ N(0, 0.02) with 0.1% of entries x10; activations ~ N(0, 1) with
              1% of the K channels x20.
  sweep       K=8192, N=28672, same distributions, M in {1, 8, 32, 128}.
  gran        K=N=8192, weights ~ N(0, 0.02) with one x20 outlier in every
              1024 consecutive K elements of each row; M in {1, 16}.
  full70b     80 layers x {qkv 8192->10240, o 8192->8192, gate+up
              8192->57344, down 28672->8192}; weights ~ N(0, 0.02).
These stand in for real checkpoints and traffic: no dataset or trained
weights are used anywhere.
"""
from __future__ import annotations

import math

import torch

WEIGHT_STD = 0.02

# Linear layers of one 70B-shaped transformer block: (name, K, N).
FULL70B_LINEARS = (("qkv", 8192, 10240), ("o", 8192, 8192), ("gate_up", 8192, 57344),
                   ("down", 28672, 8192))
FULL70B_LAYERS = 80

SEEDS = {"tiny": 0, "decode_up": 2, "sweep": 3, "gran": 4}


def full70b_seed(layer: int, j: int) -> int:
    return 5000 + layer * 4 + j


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def tiny_weight(seed: int = SEEDS["tiny"], N: int = 512, K: int = 256) -> torch.Tensor:
    """binary32 [N][K] ~ N(0, 0.02) with 4 uniformly placed entries set to +-1.0 (random sign)."""
    g = _gen(seed)
    w = torch.randn(N, K, generator=g) * WEIGHT_STD
    pos = torch.randperm(N * K, generator=g)[:4]
    sign = torch.randint(0, 2, (4,), generator=g).float() * 2 - 1
    w.view(-1)[pos] = sign
    return w


def llm_weight(N: int, K: int, seed: int, outlier_frac: float = 1e-3, outlier_mult: float = 10.0,
               dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """[N][K] ~ N(0, 0.02); a fraction of uniformly placed entries multiplied by outlier_mult."""
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device) * WEIGHT_STD
    n_out = int(round(outlier_frac * N * K))
    if n_out > 0:
        pos = torch.randint(0, N * K, (n_out,), generator=g, device=device)
        w.view(-1)[pos] *= outlier_mult
    return w.to(dtype)


def block_outlier_weight(N: int, K: int, seed: int, block: int = 1024, mult: float = 20.0,
                         dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """[N][K] ~ N(0, 0.02) with one entry x``mult`` at a uniform position in each ``block`` of K."""
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device) * WEIGHT_STD
    nb = (K + block - 1) // block
    off = torch.randint(0, block, (N, nb), generator=g, device=device)
    base = torch.arange(nb, device=device) * block
    col = (base[None, :] + off).clamp_max(K - 1)
    rows = torch.arange(N, device=device)[:, None].expand(N, nb)
    w[rows, col] *= mult
    return w.to(dtype)


def activations(M: int, K: int, seed: int, salient_frac: float = 0.01, salient_mult: float = 20.0,
                device="cpu", channel_seed: int | None = None) -> torch.Tensor:
    """bf16 [M][K] ~ N(0, 1); a random ``salient_frac`` of the K channels multiplied by salient_mult.
    With ``channel_seed`` the salient channels are fixed by it (the same channels for every ``seed``, as
    the inputs of one layer would be); without it they follow ``seed``."""
    g = _gen(seed + 1_000_003, device)
    x = torch.randn(M, K, generator=g, device=device)
    n_sal = int(round(salient_frac * K))
    if n_sal > 0:
        gc = g if channel_seed is None else _gen(channel_seed + 7_000_001, device)
        ch = torch.randperm(K, generator=gc, device=device)[:n_sal]
        x[:, ch] *= salient_mult
    return x.to(torch.bfloat16)


def wide_range_activations(M: int, K: int, seed: int, spread: float = 4.0, device="cpu") -> torch.Tensor:
    """bf16 [M][K]: N(0, 1) times exp(spread * N(0, 1)), so the values of one group span many binades
    (their binary32 sums round, which makes exact cancellation a real test)."""
    g = _gen(seed)
    x = torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, K, generator=g) * spread)
    return x.to(torch.bfloat16).to(device)


def plain_activations(M: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [M][K] ~ N(0, 1)."""
    g = _gen(seed + 2_000_003, device)
    return torch.randn(M, K, generator=g, device=device).to(torch.bfloat16)


def uniform_weight(N: int, K: int, seed: int, lo: float = -1.0, hi: float = 1.0,
                   dtype=torch.float32) -> torch.Tensor:
    """[N][K] ~ U(lo, hi)."""
    g = _gen(seed)
    return (torch.rand(N, K, generator=g) * (hi - lo) + lo).to(dtype)


def heavy_tail_weight(N: int, K: int, seed: int, dtype=torch.float32) -> torch.Tensor:
    """[N][K] Student-t-like draws: a normal divided by the root of a chi-square with 3 dof."""
    g = _gen(seed)
    z = torch.randn(N, K, generator=g)
    c = (torch.randn(N, K, 3, generator=g) ** 2).sum(-1) / 3.0
    return (z / c.sqrt() * WEIGHT_STD).to(dtype)


def offset_group_weight(N: int, K: int, seed: int, group: int = 128, dtype=torch.float32) -> torch.Tensor:
    """[N][K] ~ N(0, 0.02), except every third row, which repeats one block of `group` values along K: a
    band of width b (10^-2 to 1) whose near edge lies d from zero, on either side, with d / b log-uniform
    in [8, 300].  Every block of such a row lies on one side of zero, far from it compared with its width
    (a pattern real weights rarely show but the format allows)."""
    g = _gen(seed)
    w = torch.randn(N, K, generator=g) * WEIGHT_STD
    rows = torch.arange(0, N, 3)
    n = len(rows)
    t = torch.rand(n, group, generator=g)
    t[:, 0], t[:, 1] = 0.0, 1.0  # the band's edges are taken
    width = 10.0 ** (-2.0 * torch.rand(n, 1, generator=g))
    dist = width * 10.0 ** (math.log10(8.0) + torch.rand(n, 1, generator=g) * math.log10(300.0 / 8.0))
    sign = torch.where(torch.rand(n, 1, generator=g) < 0.5, -1.0, 1.0)
    block = sign * (dist + width * t)
    w[rows] = block.repeat(1, K // group)
    return w.to(dtype)


def positive_activations(M: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [M][K] = |N(0, 1)| + 0.05: activations of one sign, so no rounding error cancels in a sum."""
    g = _gen(seed + 3_000_017)
    return (torch.randn(M, K, generator=g).abs() + 0.05).to(torch.bfloat16).to(device)


def one_signed_weight(N: int, K: int, seed: int, dtype=torch.float32) -> torch.Tensor:
    """[N][K] strictly positive draws in every row (|N(0, 0.02)| + 0.01)."""
    g = _gen(seed)
    return (torch.randn(N, K, generator=g).abs() * WEIGHT_STD + 0.01).to(dtype)


# KV cache of one layer for the decode-attention read: [B][T][H][D] (sequences, token slots, KV heads,
# head_dim) bf16, and the decode step's queries [B][Hq][D].  The pages' geometry for the 70B model at batch
# 128 is H = 8 KV heads, Hq = 64 query heads, D = 128, 8,000-token contexts.
KV_70B = {"H": 8, "Hq": 64, "D": 128, "B": 128, "T": 8000}


def kv_cache(B: int, T: int, H: int, D: int, seed: int, offset: float = 0.0, device="cpu") -> torch.Tensor:
    """bf16 [B][T][H][D] ~ N(0, 1) (+ offset: with a large offset every vector lies on one side of zero)."""
    g = _gen(seed + 4_000_037, device)
    return (torch.randn(B, T, H, D, generator=g, device=device) + offset).to(torch.bfloat16)


def queries(B: int, Hq: int, D: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [B][Hq][D] ~ N(0, 1)."""
    g = _gen(seed + 5_000_011, device)
    return torch.randn(B, Hq, D, generator=g, device=device).to(torch.bfloat16)


def sequence_lengths(B: int, T: int, seed: int) -> torch.Tensor:
    """int32 [B] uniform in [1, T] (a mix of short and long contexts)."""
    g = _gen(seed + 6_000_001)
    return torch.randint(1, T + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def channel_scales(K: int, seed: int, spread: float = 0.5) -> torch.Tensor:
    """float32 [K] positive per-input-channel scales exp(spread * N(0, 1)) (stand-ins for the scales an
    activation-aware search produces)."""
    g = _gen(seed + 7_000_019)
    return torch.exp(torch.randn(K, generator=g) * spread).float()
