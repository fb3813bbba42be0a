"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers: it holds none of the quantization or
matmul arithmetic, so the oracle and the CUDA library can both be fed from it
without sharing any of the method's code.

The pages measure on real checkpoints and datasets (Llama-3.x, Qwen, SmolLM,
WikiText-2); none is available here, so these generators stand in for them with
the *shapes* of those models' linear layers and simple value distributions:

* weights ``W[N, K]`` fp32 ~ N(0, 0.02), NumPy PCG64; on the decode/prefill
  workloads exactly ``round(0.001 * N * K)`` positions, drawn uniformly without
  replacement from the same generator, are multiplied by 10 (outliers, the
  failure mode the "What you lose" section of "Quantizing a Model for MLX"
  describes);
* activations ``x[M, K]`` ~ N(0, 1) drawn in fp32 and rounded to bf16 (RNE).

Seeds: the tiny case uses weight seed 0; workload ``c`` (1-based, as listed in
``WORKLOADS``) shape ``i`` uses ``1000 + 100 * c + i``; activations use the
weight seed + 1.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def weights(N: int, K: int, seed: int, outliers: bool = True) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    w = rng.normal(0.0, 0.02, size=(N, K)).astype(np.float32)
    if outliers:
        n_out = int(round(0.001 * N * K))
        if n_out:
            idx = rng.choice(N * K, size=n_out, replace=False)
            w.reshape(-1)[idx] *= np.float32(10.0)
    return w


def activations(M: int, K: int, seed: int) -> torch.Tensor:
    """x ~ N(0,1) rounded to bf16; returned as a CPU bf16 tensor [M, K]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=(M, K), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a bf16 tensor (a view, no rounding)."""
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass(frozen=True)
class Case:
    name: str
    M: int
    K: int
    N: int
    bits: int
    G: int
    w_seed: int
    outliers: bool = True

    @property
    def x_seed(self) -> int:
        return self.w_seed + 1


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    cases: tuple = field(default_factory=tuple)


def _seed(c: int, i: int) -> int:
    return 1000 + 100 * c + i


def _build():
    w1 = Workload(1, "tiny W[256,512] 4-bit G64 M=1",
                  (Case("tiny", 1, 512, 256, 4, 64, 0, outliers=False),))
    llama = [(4096, 4096), (4096, 14336), (14336, 4096)]
    w2 = Workload(2, "decode QMV M=1, Llama-3-8B linears, 4-bit G64",
                  tuple(Case(f"qmv_K{K}_N{N}", 1, K, N, 4, 64, _seed(2, i)) for i, (K, N) in enumerate(llama)))
    w3 = Workload(3, "small-M decode M=1..8, K=4096 N=14336, 4-bit G64",
                  tuple(Case(f"smallm_M{M}", M, 4096, 14336, 4, 64, _seed(3, i))
                        for i, M in enumerate((1, 2, 3, 4, 5, 6, 8))))
    sweep = []
    i = 0
    for b in (2, 3, 4, 8):
        for G in (32, 64, 128):
            sweep.append(Case(f"sweep_b{b}_G{G}", 1, 8192, 28672, b, G, _seed(4, i)))
            i += 1
    w4 = Workload(4, "bits x group sweep M=1, K=8192 N=28672", tuple(sweep))
    pre = []
    i = 0
    for M in (512, 2048, 8192):
        for (K, N) in ((4096, 14336), (14336, 4096)):
            pre.append(Case(f"qmm_M{M}_K{K}_N{N}", M, K, N, 4, 64, _seed(5, i)))
            i += 1
    w5 = Workload(5, "prefill QMM M=512/2048/8192, 4-bit G64", tuple(pre))
    return (w1, w2, w3, w4, w5)


WORKLOADS = _build()


def case(name: str) -> Case:
    for wl in WORKLOADS:
        for c in wl.cases:
            if c.name == name:
                return c
    raise KeyError(name)
