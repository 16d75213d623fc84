"""Parity at the full benchmark size (Qwen3-8B-shaped target, 5-layer block-16
drafter, batch 1) in the launch configuration bench.py times.

The fp64 oracle replays two draft/verify iterations teacher-forced on the GPU's
tokens after a short prompt (a 512-token oracle prefill would take minutes on
the host): every drafter and verify logit row is compared (bf16 tolerance
3e-2), token ids must match except at oracle near-ties (top-1/top-2 margin
below 0.05), and accept lengths / commits follow the greedy rule bit for bit.
"""
import numpy as np
import pytest
import torch

import block_diffusion_speculative_layers_b200 as dfl
import oracle
from synthetic import get_config, make_prompt, make_weight
from synthetic.fast import make_weights_host

from parity import replay

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def full_pair():
    cfg = get_config("qwen3_8b")
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=256, keep_logits=True)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    spec = oracle.OracleSpec(cfg, make_weights_host(cfg))
    yield cfg, gpu, spec
    gpu.close()


def test_qwen3_8b_shape_replay(cuda_device, full_pair):
    cfg, gpu, spec = full_pair
    prompt = make_prompt("zipf", 24, cfg.target.vocab, cfg.seed)
    rep = replay(gpu, spec, cfg, [prompt], 2, 3e-2, 0.05)
    print(f"max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
    assert rep.mismatches_outside_ties == 0, rep
    assert rep.max_dlogit <= 3e-2, rep.max_dlogit
