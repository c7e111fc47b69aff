"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module only draws random numbers and rounds them to the storage dtype
(BF16 for weights and activations, FP32 for the activation-scale vector).  It
holds none of the DV-SSQ arithmetic: no rotation, no quantisation, no
selection.  Both the CUDA path and the fp64 oracle consume exactly these
tensors.

Workload recipes (shapes and value distributions) follow the two F-Labs model
cards: "Spark-X2.5-4B-Hadamard-GSQ" (hidden 2560, intermediate 10240, 36
layers, H_256 blocks, Tier A/B/C) and "MiniCPM5-2B-Hadamard-GSQ" (hidden 2048,
H_128 blocks, ranks 16/24/32).  The pages ship no weights and no prompts, so
weights are N(0, 0.02) with a few scaled "outlier" input columns and
activations are N(0, 1) with a few scaled outlier channels.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

__all__ = [
    "weight", "weight_device", "act_scale", "activations", "lowrank_factors", "Workload",
    "WORKLOADS", "layer_seed", "stack_rank",
]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def weight(M: int, K: int, seed: int, std: float = 0.02,
           n_outlier_cols: int = 0, outlier_scale: float = 1.0) -> torch.Tensor:
    """W [M][K] BF16 ~ N(0, std); ``n_outlier_cols`` input columns scaled."""
    g = _rng(seed)
    w = g.standard_normal((M, K), dtype=np.float32) * np.float32(std)
    if n_outlier_cols:
        cols = g.choice(K, size=n_outlier_cols, replace=False)
        w[:, cols] *= np.float32(outlier_scale)
    return _to_bf16(w)


def weight_device(M: int, K: int, seed: int, device, std: float = 0.02,
                  n_outlier_cols: int = 0, outlier_scale: float = 1.0) -> torch.Tensor:
    """Like ``weight`` but drawn on ``device`` by torch's seeded generator.

    For workloads too large to draw on the host in reasonable time (the
    36-layer stack); the values differ from ``weight``'s for the same seed.
    """
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn((M, K), generator=g, device=device, dtype=torch.float32) * std
    if n_outlier_cols:
        cols = torch.randperm(K, generator=g, device=device)[:n_outlier_cols]
        w[:, cols] *= outlier_scale
    return w.to(torch.bfloat16)


def act_scale(K: int, seed: int) -> torch.Tensor:
    """Per-input-channel activation scale |N(0,1)| + 0.1, FP32 [K]."""
    g = _rng(seed)
    return torch.from_numpy(np.abs(g.standard_normal(K, dtype=np.float32))
                            + np.float32(0.1))


def activations(T: int, K: int, seed: int, n_outlier: int = 0,
                outlier_scale: float = 1.0) -> torch.Tensor:
    """x [T][K] BF16 ~ N(0,1) with ``n_outlier`` channels scaled."""
    g = _rng(seed)
    x = g.standard_normal((T, K), dtype=np.float32)
    if n_outlier:
        ch = g.choice(K, size=n_outlier, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    return _to_bf16(x)


def lowrank_factors(M: int, K: int, r: int, seed: int, std: float = 0.01):
    """Stand-in BF16 factors U [M][r], V [r][K] with a residual-like scale.

    Used where the factor values do not affect the measured work (timing);
    parity checks use the oracle's truncated-SVD factors instead.
    """
    g = _rng(seed)
    U = g.standard_normal((M, r), dtype=np.float32) * np.float32(std)
    V = g.standard_normal((r, K), dtype=np.float32) * np.float32(std)
    return _to_bf16(U), _to_bf16(V)


def stack_rank(layer: int) -> int:
    """Residual rank of a layer of the 36-layer Spark stack: 24 on layers
    14..28, 16 elsewhere."""
    return 24 if 14 <= layer <= 28 else 16


def layer_seed(base: int, layer: int, which: int) -> int:
    """Per-matrix seed of the 36-layer stack: which = 0 gate, 1 up, 2 down."""
    return base * 1000 + layer * 3 + which


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    block: int
    rank: int
    tokens: tuple
    w_outlier_cols: int
    w_outlier_scale: float
    x_outliers: int
    x_outlier_scale: float
    seed: int

    @property
    def n_sal(self) -> int:
        # top 12.5 % of the input channels (Tier A)
        return self.K // 8

    def weight(self, seed_offset: int = 0) -> torch.Tensor:
        return weight(self.M, self.K, self.seed + seed_offset,
                      n_outlier_cols=self.w_outlier_cols,
                      outlier_scale=self.w_outlier_scale)

    def act_scale(self, seed_offset: int = 0) -> torch.Tensor:
        return act_scale(self.K, self.seed + 7919 + seed_offset)

    def activations(self, T: int, seed_offset: int = 0) -> torch.Tensor:
        return activations(T, self.K, self.seed + 104729 + 31 * T + seed_offset,
                           n_outlier=self.x_outliers,
                           outlier_scale=self.x_outlier_scale)


WORKLOADS = {
    # 256x512 single layer, 4 outlier input columns x20, 2 outlier channels x30
    "tiny": Workload("tiny", 256, 512, 256, 8, (4,), 4, 20.0, 2, 30.0, 0),
    # Spark-shaped down_proj 2560x10240: 0.1 % columns x15, 0.5 % channels x25
    "spark_down": Workload("spark_down", 2560, 10240, 256, 16, (1, 16),
                           10, 15.0, 51, 25.0, 1),
    # MiniCPM-shaped k_proj-like and up_proj-like layers, hidden 2048, H_128
    "minicpm_k": Workload("minicpm_k", 512, 2048, 128, 32, (1, 8, 64),
                          0, 1.0, 10, 25.0, 2),
    "minicpm_up": Workload("minicpm_up", 8192, 2048, 128, 24, (1, 8, 64),
                           0, 1.0, 10, 25.0, 3),
    # Spark up_proj 10240x2560 driven with a 4096-token prefill
    "spark_up_prefill": Workload("spark_up_prefill", 10240, 2560, 256, 16,
                                 (4096,), 3, 15.0, 13, 25.0, 4),
    # one gate/up and one down matrix of the 36-layer Spark MLP stack
    "spark_gate": Workload("spark_gate", 10240, 2560, 256, 16, (1,),
                           0, 1.0, 13, 25.0, 5),
}
