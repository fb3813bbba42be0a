"""Cached synthetic inputs and oracle results for the GPU parity tests."""
from __future__ import annotations

import functools

import numpy as np

import oracle
import synth


@functools.lru_cache(maxsize=2)
def weights(N: int, K: int, seed: int, outliers: bool = True) -> np.ndarray:
    return synth.weights(N, K, seed, outliers)


@functools.lru_cache(maxsize=2)
def quantized(N: int, K: int, seed: int, outliers: bool, G: int, bits: int):
    return oracle.quantize(weights(N, K, seed, outliers), G, bits)


def activations_bits(M: int, K: int, seed: int) -> np.ndarray:
    return synth.bf16_bits(synth.activations(M, K, seed))


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """A seeded sample of output rows (tokens) that always includes the first and last."""
    if M <= n:
        return np.arange(M)
    rng = np.random.Generator(np.random.PCG64(seed))
    mid = rng.choice(np.arange(1, M - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, M - 1], mid]))
