"""Seeded synthetic workloads for the BinaryAttention forward pass.

This module only draws random numbers: it holds none of the method's arithmetic, so
both the CUDA path and the CPU oracle can take their inputs from it. Every tensor is
generated on the CPU with a seeded ``torch.Generator`` and is bit-for-bit
reproducible for a given torch version.

The shapes stand in for the workloads the pages evaluate on (ImageNet classification
with DeiT-B, DiT-XL/2 generation at 256/512/1024 px, and a long-sequence sweep); no
dataset or trained weight is used or needed.

Readings of the workload descriptions (stated once here):
  * "N(0, s)" is read as mean 0 and standard deviation s.
  * DeiT-B outliers: per head, 4 distinct channels are drawn independently for q and
    for k, and those channels are multiplied by 8 for every batch and token.
  * DiT-XL/2-256 offsets: one offset per (head, channel), drawn separately for q and
    for k, shared over batch and tokens.
  * Heavy tails: each entry is, with probability 0.02, replaced by a Student-t draw
    with 3 degrees of freedom, built as z / sqrt(chi2_3 / 3) from the same generator.
  * Relative-position tables are centred: a table with half-extents (th, tw) serves a
    grid of gh <= th rows and gw <= tw columns. Non-square sweep lengths use a 1:2 grid.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

BIAS_NONE, BIAS_DENSE, BIAS_RELPOS2D = 0, 1, 2


@dataclass
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: torch.dtype
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    bias_kind: int = BIAS_NONE
    bias: Optional[torch.Tensor] = None  # dense [H,N,N] fp32, or table [H,(2th-1)(2tw-1)] fp32
    batch_stride: int = 0
    grid_h: int = 0
    grid_w: int = 0
    table_h: int = 0
    table_w: int = 0
    n_prefix: int = 0
    seed: int = 0
    meta: Dict[str, str] = field(default_factory=dict)

    @property
    def dtype_name(self) -> str:
        return {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[self.dtype]


def _normal(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32) * std


def _student_t3(g: torch.Generator, shape) -> torch.Tensor:
    z = torch.randn(shape, generator=g, dtype=torch.float32)
    chi2 = (torch.randn((3,) + tuple(shape), generator=g, dtype=torch.float32) ** 2).sum(0)
    return z / torch.sqrt(chi2 / 3.0)


def _heavy_tailed(g: torch.Generator, shape, p: float = 0.02) -> torch.Tensor:
    x = _normal(g, shape)
    mask = torch.rand(shape, generator=g) < p
    t = _student_t3(g, shape)
    return torch.where(mask, t, x)


def _with_outliers(g: torch.Generator, x: torch.Tensor, n_ch: int = 4, factor: float = 8.0) -> torch.Tensor:
    B, H, N, d = x.shape
    scale = torch.ones(H, d)
    for h in range(H):
        ch = torch.randperm(d, generator=g)[:n_ch]
        scale[h, ch] = factor
    return x * scale.view(1, H, 1, d)


def relpos_grid(N: int):
    """1:2 (or square) grid for a sweep length N: gh = 2^floor(log2(N)/2), gw = N/gh."""
    gh = 2 ** int(math.floor(math.log2(N) / 2))
    return gh, N // gh


def tiny(seed: int = 0) -> Workload:
    """B=1 H=1 N=256 d=64 fp16, q,k,v ~ N(0,1), dense bias [1,256,256] ~ N(0,0.1)."""
    g = torch.Generator().manual_seed(seed)
    B, H, N, d = 1, 1, 256, 64
    q, k, v = (_normal(g, (B, H, N, d)) for _ in range(3))
    bias = _normal(g, (H, N, N), 0.1)
    return Workload("tiny_b1_h1_n256_d64", B, H, N, d, torch.float16, q.half(), k.half(), v.half(),
                    BIAS_DENSE, bias, 0, seed=seed)


def deit_b(seed: int = 1, B: int = 64) -> Workload:
    """DeiT-B 224px shape: B=64 H=12 N=197 (14x14 grid + CLS) d=64 fp16, q,k with 4
    outlier channels per head (x8), rel-pos table [12, 27^2] ~ N(0,0.02), CLS bias 0."""
    g = torch.Generator().manual_seed(seed)
    H, N, d = 12, 197, 64
    q = _with_outliers(g, _normal(g, (B, H, N, d)))
    k = _with_outliers(g, _normal(g, (B, H, N, d)))
    v = _normal(g, (B, H, N, d))
    table = _normal(g, (H, 27 * 27), 0.02)
    return Workload(f"deit_b_b{B}_h12_n197_d64", B, H, N, d, torch.float16, q.half(), k.half(), v.half(),
                    BIAS_RELPOS2D, table, 0, 14, 14, 14, 14, 1, seed)


def dit_xl2_256(seed: int = 2, B: int = 32) -> Workload:
    """DiT-XL/2 256px shape: B=32 H=16 N=256 d=72 bf16, q,k = N(0,1) + per-(head,channel)
    offset ~ N(0,0.5), dense bias [16,256,256] ~ N(0,0.1) broadcast over the batch."""
    g = torch.Generator().manual_seed(seed)
    H, N, d = 16, 256, 72
    q = _normal(g, (B, H, N, d)) + _normal(g, (1, H, 1, d), 0.5)
    k = _normal(g, (B, H, N, d)) + _normal(g, (1, H, 1, d), 0.5)
    v = _normal(g, (B, H, N, d))
    bias = _normal(g, (H, N, N), 0.1)
    return Workload(f"dit_xl2_256_b{B}_h16_n256_d72", B, H, N, d, torch.bfloat16, q.bfloat16(),
                    k.bfloat16(), v.bfloat16(), BIAS_DENSE, bias, 0, seed=seed)


def dit_highres(N: int = 1024, B: Optional[int] = None, seed: int = 3) -> Workload:
    """DiT-XL/2 512px (N=1024, B=8) or 1024px (N=4096, B=2) shape, d=64 bf16, q,k,v ~ N(0,1)
    with 2% Student-t(3) entries, rel-pos table [16,127^2] ~ N(0,0.02) (half-extent 64)."""
    if B is None:
        B = {1024: 8, 4096: 2}[N]
    g = torch.Generator().manual_seed(seed)
    H, d = 16, 64
    q, k, v = (_heavy_tailed(g, (B, H, N, d)) for _ in range(3))
    table = _normal(g, (H, 127 * 127), 0.02)
    side = int(round(math.sqrt(N)))
    assert side * side == N
    return Workload(f"dit_{'512' if N == 1024 else '1024'}_b{B}_h16_n{N}_d64", B, H, N, d, torch.bfloat16,
                    q.bfloat16(), k.bfloat16(), v.bfloat16(), BIAS_RELPOS2D, table, 0, side, side, 64, 64, 0,
                    seed)


def sweep(N: int, d: int = 64, seed: int = 4, H: int = 16) -> Workload:
    """Long-sequence sweep: B=1 H=16 d in {64,128} bf16, q,k,v ~ N(0,1), rel-pos table
    sized for a gh x gw grid (gh = 2^floor(log2 N / 2))."""
    g = torch.Generator().manual_seed(seed)
    B = 1
    gh, gw = relpos_grid(N)
    q, k, v = (_normal(g, (B, H, N, d)) for _ in range(3))
    table = _normal(g, (H, (2 * gh - 1) * (2 * gw - 1)), 0.02)
    return Workload(f"sweep_b1_h{H}_n{N}_d{d}", B, H, N, d, torch.bfloat16, q.bfloat16(), k.bfloat16(),
                    v.bfloat16(), BIAS_RELPOS2D, table, 0, gh, gw, gh, gw, 0, seed)


SWEEP_N: List[int] = [1024, 2048, 4096, 8192, 16384, 32768]


def by_name(name: str) -> Workload:
    """Look a workload up by a short name: tiny, deit_b, dit256, dit512, dit1024,
    sweep<N>_d<d> (e.g. sweep4096_d64)."""
    if name == "tiny":
        return tiny()
    if name == "deit_b":
        return deit_b()
    if name == "dit256":
        return dit_xl2_256()
    if name == "dit512":
        return dit_highres(1024)
    if name == "dit1024":
        return dit_highres(4096)
    if name.startswith("sweep"):
        n_part, d_part = name[len("sweep"):].split("_d")
        return sweep(int(n_part), int(d_part))
    raise KeyError(name)


def random_case(B: int, H: int, N: int, d: int, dtype=torch.float16, bias_kind: int = BIAS_NONE,
                seed: int = 0, grid=None, n_prefix: int = 0, batch_bias: bool = False) -> Workload:
    """Small random case for edge-shape tests (ragged N, odd d, tails)."""
    g = torch.Generator().manual_seed(seed)
    q, k, v = (_normal(g, (B, H, N, d)) for _ in range(3))
    w = Workload(f"case_b{B}_h{H}_n{N}_d{d}", B, H, N, d, dtype, q.to(dtype), k.to(dtype), v.to(dtype),
                 seed=seed)
    if bias_kind == BIAS_DENSE:
        if batch_bias:
            w.bias = _normal(g, (B, H, N, N), 0.1)
            w.batch_stride = H * N * N
        else:
            w.bias = _normal(g, (H, N, N), 0.1)
        w.bias_kind = BIAS_DENSE
    elif bias_kind == BIAS_RELPOS2D:
        gh, gw = grid if grid is not None else (1, N - n_prefix)
        th, tw = gh, gw
        w.bias = _normal(g, (H, (2 * th - 1) * (2 * tw - 1)), 0.05)
        w.bias_kind = BIAS_RELPOS2D
        w.grid_h, w.grid_w, w.table_h, w.table_w, w.n_prefix = gh, gw, th, tw, n_prefix
    return w
