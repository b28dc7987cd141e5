"""Seeded synthetic inputs shaped like the pages' NVFP4 W4A4 workloads.

This module only draws random numbers; it holds none of the quantizer's or
the GEMM's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.  Everything is generated on the CPU with
``torch.Generator().manual_seed(seed)`` in float32 and cast to bfloat16 once,
so every consumer sees identical bytes.

Shapes stand in for linear layers of the model families the pages evaluate
(Four-Over-Six summary, "사전 학습" / "학습 후 양자화" sections: Llama / Qwen
layers; Minima page "산업 영향" section: a 27B hybrid model; ARCQuant summary,
"실험 결과" section: Llama-3.1-8B).  No model weights or datasets are used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

CHUNK_ROWS = 2048  # bounded temporaries when drawing large tensors


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed)


def normal(rows: int, cols: int, std: float, seed: int) -> torch.Tensor:
    """i.i.d. N(0, std^2), float32."""
    g = _gen(seed)
    out = torch.empty(rows, cols, dtype=torch.float32)
    for r0 in range(0, rows, CHUNK_ROWS):
        r1 = min(rows, r0 + CHUNK_ROWS)
        out[r0:r1] = torch.randn(r1 - r0, cols, generator=g) * std
    return out


def student_t(rows: int, cols: int, nu: int, scale: float, seed: int) -> torch.Tensor:
    """scale * T_nu with integer nu: z / sqrt(sum_{i<nu} z_i^2 / nu)."""
    g = _gen(seed)
    out = torch.empty(rows, cols, dtype=torch.float32)
    for r0 in range(0, rows, CHUNK_ROWS):
        r1 = min(rows, r0 + CHUNK_ROWS)
        z = torch.randn(r1 - r0, cols, generator=g)
        chi2 = torch.zeros_like(z)
        for _ in range(nu):
            chi2.add_(torch.randn(r1 - r0, cols, generator=g).square_())
        out[r0:r1] = z.div_(chi2.div_(nu).sqrt_()).mul_(scale)
    return out


def outlier_channels(x: torch.Tensor, frac: float, mult: float, seed: int) -> torch.Tensor:
    """Multiply round(frac * K) columns (chosen by randperm over K) by mult in
    every row: channel-structured activation outliers."""
    K = x.shape[1]
    n = max(1, round(frac * K))
    idx = torch.randperm(K, generator=_gen(seed))[:n]
    x[:, idx] *= mult
    return x


def outlier_entries(x: torch.Tensor, frac: float, mult: float, seed: int) -> torch.Tensor:
    """Multiply exactly round(frac * numel) entries (chosen by randperm) by mult."""
    flat = x.view(-1)
    n = round(frac * flat.numel())
    idx = torch.randperm(flat.numel(), generator=_gen(seed))[:n]
    flat[idx] *= mult
    return x


@dataclass(frozen=True)
class Operand:
    rows: int
    K: int
    dist: str                # "normal" | "t"
    param: float             # std for normal, nu for t
    scale: float = 1.0       # multiplier for t
    outliers: str = ""       # "" | "entries" | "channels"
    out_frac: float = 0.0
    out_mult: float = 1.0
    seed: int = 0

    def make(self) -> torch.Tensor:
        if self.dist == "normal":
            x = normal(self.rows, self.K, self.param, self.seed)
        elif self.dist == "t":
            x = student_t(self.rows, self.K, int(self.param), self.scale, self.seed)
        else:
            raise ValueError(self.dist)
        if self.outliers == "entries":
            outlier_entries(x, self.out_frac, self.out_mult, self.seed + 1000)
        elif self.outliers == "channels":
            outlier_channels(x, self.out_frac, self.out_mult, self.seed + 1000)
        return x.to(torch.bfloat16)

    @property
    def numel(self) -> int:
        return self.rows * self.K


@dataclass(frozen=True)
class Workload:
    name: str
    x: Operand
    w: Operand | None
    # quantization recipes: (mode, rule, fp8_max) for X and W
    x_recipes: tuple = ()
    w_recipe: tuple | None = None
    note: str = ""

    @property
    def M(self):
        return self.x.rows

    @property
    def K(self):
        return self.x.K

    @property
    def N(self):
        return self.w.rows if self.w else 0

    @property
    def gemm_flops(self):
        return 2 * self.M * self.N * self.K


# mode / rule names as the C ABI spells them
SIX, FOUR_OVER_SIX = "six", "four_over_six"
MAX, MAE, MSE = "max", "mae", "mse"

WORKLOADS = {
    # X 64x512 ~N(0,1) with 1 % of entries x20, W 256x512 ~N(0,0.02), seed 0
    "pr1": Workload(
        "pr1",
        Operand(64, 512, "normal", 1.0, outliers="entries", out_frac=0.01, out_mult=20.0, seed=0),
        Operand(256, 512, "normal", 0.02, seed=1),
        x_recipes=((SIX, MAX, 448.0), (FOUR_OVER_SIX, MSE, 256.0)),
        w_recipe=(SIX, MAX, 448.0),
        note="PR1 reference case: scale-6 (F=448) and 4/6-MSE (F=256) on both operands",
    ),
    # 8B-dense-shaped MLP up-projection
    "mlp8b": Workload(
        "mlp8b",
        Operand(4096, 4096, "normal", 1.0, outliers="channels", out_frac=0.005, out_mult=50.0, seed=0),
        Operand(14336, 4096, "normal", 0.02, seed=1),
        x_recipes=((FOUR_OVER_SIX, MSE, 256.0),),
        w_recipe=(SIX, MAX, 448.0),
        note="4/6-MSE on activations only, scale-6 weights",
    ),
    # 27B-hybrid-shaped linear-attention projection (gate/QKV)
    "attn27b": Workload(
        "attn27b",
        Operand(8192, 5120, "t", 4, scale=1.0, seed=0),
        Operand(12288, 5120, "normal", 0.015, seed=1),
        x_recipes=((FOUR_OVER_SIX, MAE, 256.0),),
        w_recipe=(FOUR_OVER_SIX, MAE, 256.0),
        note="full W4A4 with 4/6-MAE on both operands",
    ),
    # long-prefill MLP: the largest GEMM
    "prefill": Workload(
        "prefill",
        Operand(32768, 5120, "normal", 1.0, outliers="channels", out_frac=0.002, out_mult=100.0, seed=0),
        Operand(17408, 5120, "normal", 0.015, seed=1),
        x_recipes=((SIX, MAX, 448.0), (FOUR_OVER_SIX, MSE, 256.0)),
        w_recipe=(SIX, MAX, 448.0),
        note="quantize X per call (scale-6 vs 4/6-MSE) then GEMM with pre-quantized W",
    ),
}

# quantize-only sweep: 0.5 * Student-t(nu=3), 0.5 % of columns x50 in every row
SWEEP_SHAPES = ((4096, 4096), (8192, 8192), (16384, 16384), (32768, 16384))
SWEEP_RECIPES = ((SIX, MAX, 448.0), (FOUR_OVER_SIX, MAX, 256.0),
                 (FOUR_OVER_SIX, MAE, 256.0), (FOUR_OVER_SIX, MSE, 256.0))


def sweep_operand(rows: int, K: int, seed: int = 0) -> Operand:
    return Operand(rows, K, "t", 3, scale=0.5, outliers="channels", out_frac=0.005,
                   out_mult=50.0, seed=seed)


def small_operand(rows: int, K: int, seed: int, kind: str = "t") -> Operand:
    """Small parity-test operands with the sweep's value distribution."""
    if kind == "t":
        return sweep_operand(rows, K, seed)
    return Operand(rows, K, "normal", 1.0, outliers="entries", out_frac=0.01, out_mult=20.0,
                   seed=seed)


def sample_rows(rows: int, n: int, seed: int) -> torch.Tensor:
    """About n distinct sorted row indices for sampled full-size parity
    checks, always including the first and the last row."""
    n = max(2, min(n, rows))
    idx = torch.randperm(rows, generator=_gen(seed))[: n - 2]
    return torch.unique(torch.cat([idx, torch.tensor([0, rows - 1])]))
