"""Host-side plumbing of data-parallel replicas (one process per GPU).

The decode step does not shard inside a sequence: every rank holds the whole
model and decodes its own sequences, with no collective on the data path.
Ranks meet only to agree on timing and totals: the step time of the job is the
slowest rank's, the token count the sum over ranks.
"""
from __future__ import annotations

from typing import List

import numpy as np
import torch


def rank_prompt_seeds(base_seed: int, rank: int, batch: int) -> List[int]:
    """Seeds of the `batch` prompts of one rank; distinct across ranks (< 1000 per rank)."""
    if batch > 1000:
        raise ValueError("at most 1000 sequences per rank")
    return [base_seed + 1000 * rank + i for i in range(batch)]


def reduce_step(pg, ms: float, tokens: int, device) -> tuple:
    """(max over ranks of ms, sum over ranks of tokens); (ms, tokens) without a group."""
    if pg is None:
        return ms, tokens
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    n = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    pg.all_reduce(n)
    return float(t.item()), int(round(n.item()))


def reduce_max(pg, value: float, device) -> float:
    """Max over ranks (a job's time is its slowest rank's)."""
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


__all__ = ["rank_prompt_seeds", "reduce_step", "reduce_max", "np"]
