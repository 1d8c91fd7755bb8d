"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the quantization method: it only draws
bf16 activations and weights with the distributions of the workloads below
(Llama-shaped linear layers; no dataset and no trained weights are used).
Both the CUDA path and the CPU oracle receive the same tensors from here.

Recipe, per workload (one CPU ``torch.Generator`` seeded once, draws in this
order): W ~ N(0, 0.02) of shape [N, K] in fp32; X ~ N(0, 1) of shape
[M_max, K] in fp32; if the workload has outlier channels, ``randperm(K)``'s
first ``n_outliers`` columns of X are multiplied by 20; both are then rounded
to bf16 (round to nearest even).  Smaller M of the same workload take the
first M rows of X.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

GROUP = 64


@dataclass(frozen=True)
class Workload:
    name: str
    Ms: tuple
    N: int
    K: int
    seed: int
    n_outliers: int = 0
    outlier_scale: float = 20.0
    w_std: float = 0.02
    note: str = field(default="", compare=False)

    @property
    def M_max(self) -> int:
        return max(self.Ms)


WORKLOADS = {
    "tiny": Workload("tiny", (16,), 256, 512, seed=0,
                     note="tiny W4A8 GEMM, 16x256x512, no outliers"),
    "decode": Workload("decode", (1, 4, 16), 4096, 4096, seed=1, n_outliers=8,
                       note="attention-projection decode layer, N=K=4096, 8 outlier channels x20"),
    "prefill": Workload("prefill", (4096,), 4096, 4096, seed=2,
                        note="square prefill layer 4096^3, no outliers"),
    "mlp_up": Workload("mlp_up", (16, 256, 4096), 14336, 4096, seed=3, n_outliers=41,
                       note="MLP up/gate layer N=14336, K=4096, 1% outlier channels x20"),
    "down_sweep": Workload("down_sweep", tuple(2 ** i for i in range(14)), 4096, 14336, seed=4,
                           n_outliers=143,
                           note="MLP down-projection sweep M=1..8192, N=4096, K=14336, "
                                "1% outlier channels x20"),
}


def make_weights(N: int, K: int, seed: int, std: float = 0.02, gen: torch.Generator | None = None):
    g = gen if gen is not None else torch.Generator().manual_seed(seed)
    return (torch.randn(N, K, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def make_activations(M: int, K: int, seed: int, n_outliers: int = 0, outlier_scale: float = 20.0,
                     gen: torch.Generator | None = None):
    g = gen if gen is not None else torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if n_outliers:
        idx = torch.randperm(K, generator=g)[:n_outliers]
        x[:, idx] *= outlier_scale
    return x.to(torch.bfloat16)


def make_workload(w: Workload):
    """Returns (X bf16 [M_max, K], W bf16 [N, K]) on the CPU, drawn W first."""
    g = torch.Generator().manual_seed(w.seed)
    W = make_weights(w.N, w.K, w.seed, w.w_std, gen=g)
    X = make_activations(w.M_max, w.K, w.seed, w.n_outliers, w.outlier_scale, gen=g)
    return X, W


def make_problem(M: int, N: int, K: int, seed: int, n_outliers: int = 0):
    """Free-form problem with the same recipe (used for ragged and edge-case tests)."""
    g = torch.Generator().manual_seed(seed)
    W = make_weights(N, K, seed, gen=g)
    X = make_activations(M, K, seed, n_outliers, gen=g)
    return X, W


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (for the CPU oracle)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
