"""Seeded synthetic prompts (token ids), drawn on the host with numpy PCG64.

Zipf(1.1): rank r in [1, V] with probability proportional to r^-1.1, token id
r - 1 (so low ids are frequent, like a tokenizer's common tokens).  Uniform:
ids uniform in [0, V).  They stand in for the pages' benchmark prompts
(MATH-500, HumanEval, GSM8K, SPEED-Bench), which are not used here.
"""
from __future__ import annotations

import numpy as np


def zipf_prompt(n: int, vocab: int, seed: int, exponent: float = 1.1) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    p = ranks ** (-exponent)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def uniform_prompt(n: int, vocab: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def make_prompt(kind: str, n: int, vocab: int, seed: int) -> np.ndarray:
    if kind == "zipf":
        return zipf_prompt(n, vocab, seed)
    if kind == "uniform":
        return uniform_prompt(n, vocab, seed)
    raise ValueError(kind)
