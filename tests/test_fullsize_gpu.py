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


def test_qwen3_8b_shape_batch4_ragged_prompts(cuda_device, full_pair):
    """Batch-sweep shape (independent sequences in one pass; 64 verify rows):
    four sequences with different prompt lengths decode together."""
    cfg, _, spec = full_pair
    gpu = dfl.DFlash(cfg, max_batch=4, max_len=256, keep_logits=True)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    try:
        prompts = [make_prompt("zipf", n, cfg.target.vocab, cfg.seed + 3 + i) for i, n in enumerate((20, 24, 17, 30))]
        rep = replay(gpu, spec, cfg, prompts, 1, 3e-2, 0.05)
        print(f"batch 4: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    finally:
        gpu.close()


def test_llama31_8b_shape_replay(cuda_device):
    """Llama-3.1-8B shape: 32 layers, FFN 14336, vocab 128256, RoPE theta 5e5."""
    cfg = get_config("llama31_8b")
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=256, keep_logits=True)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    try:
        spec = oracle.OracleSpec(cfg, make_weights_host(cfg))
        prompt = make_prompt("uniform", 20, cfg.target.vocab, cfg.seed)
        rep = replay(gpu, spec, cfg, [prompt], 1, 3e-2, 0.05)
        print(f"llama shape: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    finally:
        gpu.close()
        torch.cuda.empty_cache()


def test_qwen3_coder_moe_shape_two_layers(cuda_device):
    """Qwen3-Coder-30B-A3B widths (hidden 2048, 32 q / 4 kv heads, 128 experts,
    top-8, expert FFN 768, vocab 151936) with two target layers."""
    from synthetic.configs import shrink
    cfg = shrink(get_config("qwen3_coder_30b_a3b"), target_layers=2, drafter_layers=1)
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=128, keep_logits=True)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    try:
        spec = oracle.OracleSpec(cfg, make_weights_host(cfg))
        prompt = make_prompt("zipf", 16, cfg.target.vocab, cfg.seed)
        rep = replay(gpu, spec, cfg, [prompt], 2, 3e-2, 0.05)
        print(f"moe shape: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    finally:
        gpu.close()
        torch.cuda.empty_cache()


def test_long_context_8192_tokens(cuda_device):
    """Long-reasoning context length (8192-token prompt, chunked prefill, split-KV
    attention over 8K keys) on a narrow bf16 model the oracle replays quickly."""
    from test_parity_gpu import tiny_cfg
    cfg = tiny_cfg(dtype="bf16", block=16, hidden=512, nq=8, nkv=2, hd=128, vocab=4096)
    spec = oracle.OracleSpec(cfg, make_weights_host(cfg))
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=8192 + 64, keep_logits=True)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    try:
        prompt = make_prompt("uniform", 8192, cfg.target.vocab, 4)
        rep = replay(gpu, spec, cfg, [prompt], 2, 3e-2, 0.05)
        print(f"8K context: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    finally:
        gpu.close()
