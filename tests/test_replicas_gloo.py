"""Data-parallel replicas on CPU: two gloo ranks agree on the job's step time
(the slowest rank's) and token count (the sum), and decode disjoint sequences.
No GPU: the collective plumbing of `bench.py --gpus N` runs here as it does
over NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_diffusion_speculative_layers_b200.replicas import rank_prompt_seeds, reduce_max, reduce_step
from synthetic import get_config, make_prompt


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [4.0, 7.5][rank]
        tokens = [100, 37][rank]
        ms_max, tok = reduce_step(dist, ms, tokens, "cpu")
        e2e = reduce_max(dist, [2.0, 1.0][rank], "cpu")
        cfg = get_config("tiny")
        seeds = rank_prompt_seeds(cfg.seed, rank, 3)
        prompts = [make_prompt("uniform", 8, cfg.target.vocab, s) for s in seeds]
        out[rank] = (ms_max, tok, e2e, seeds, [p.tolist() for p in prompts])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_partition():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 7.5          # job time = slowest rank
    assert r0[1] == r1[1] == 137          # tokens summed over ranks
    assert r0[2] == r1[2] == 2.0
    assert not set(r0[3]) & set(r1[3])    # disjoint prompt seeds
    assert r0[4] != r1[4]


def test_single_process_is_identity():
    assert reduce_step(None, 3.0, 11, "cpu") == (3.0, 11)
    assert reduce_max(None, 2.5, "cpu") == 2.5
    assert rank_prompt_seeds(5, 0, 2) == [5, 6]
    with pytest.raises(ValueError):
        rank_prompt_seeds(0, 0, 1001)
