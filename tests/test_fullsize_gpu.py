"""Parity at the full benchmark size (Qwen3-8B-shaped target, 5-layer block-16
drafter, batch 1) in the launch configuration bench.py times, and at the full
widths of the other configurations.

The fp64 oracle replays draft/verify iterations teacher-forced on the GPU's
tokens: every drafter and verify logit row is compared (bf16 tolerance 3e-2),
token ids must match except at oracle near-ties (top-1/top-2 margin below
0.05), and accept lengths / commits follow the greedy rule bit for bit.
Where a case needs a long prompt or many sequences, the model keeps its full
widths (hidden, heads, FFN, vocabulary, experts) with fewer layers, so the
oracle's prefill stays within seconds.
"""
import numpy as np
import pytest
import torch

import block_diffusion_speculative_layers_b200 as dfl
import oracle
from synthetic import get_config, make_prompt, make_weight
from synthetic.fast import make_weights_host

from parity import replay, replay_forced
from synthetic.configs import shrink

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


def test_qwen3_8b_shape_forced_accept_lengths(cuda_device, full_pair):
    """Full acceptance and partial acceptance at full size: the caller's drafts
    are the oracle's own greedy continuation, made wrong after k drafts, for
    k = 15 (all 16 tokens committed), 7, 3 and 0.  Committed tokens, accept
    lengths and new lengths bit for bit; target K/V of the committed positions
    and the drafter context K/V injected for them against the oracle's."""
    cfg, gpu, spec = full_pair
    prompt = make_prompt("zipf", 24, cfg.target.vocab, cfg.seed + 1)
    rep = replay_forced(gpu, spec, cfg, prompt, (15, 7, 3, 0), 3e-2, 0.05)
    print(f"forced: accepts {rep.accepts}, max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}")
    assert rep.mismatches_outside_ties == 0, rep
    assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    assert rep.accepts[0] == 15 or rep.near_ties > 0


def _widths_pair(name, max_batch, max_len, target_layers=2, drafter_layers=1):
    cfg = shrink(get_config(name), target_layers=target_layers, drafter_layers=drafter_layers)
    gpu = dfl.DFlash(cfg, max_batch=max_batch, max_len=max_len, keep_logits=True)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    spec = oracle.OracleSpec(cfg, make_weights_host(cfg))
    return cfg, gpu, spec


@pytest.mark.parametrize("batch,iters", [(8, 2), (32, 1)])
def test_qwen3_8b_widths_batch_sweep(cuda_device, batch, iters):
    """Batch-sweep shapes: 8 and 32 sequences of the Qwen3-8B widths decode
    together (128 and 512 verify rows, 256 and 1024 drafter QKV rows), ragged
    prompts, two target layers and one drafter layer."""
    cfg, gpu, spec = _widths_pair("qwen3_8b_sweep", batch, 96)
    try:
        prompts = [make_prompt("zipf", 4 + (7 * i) % 29, cfg.target.vocab, cfg.seed + i) for i in range(batch)]
        rep = replay(gpu, spec, cfg, prompts, iters, 3e-2, 0.05)
        print(f"batch {batch}: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    finally:
        gpu.close()
        torch.cuda.empty_cache()


def test_qwen3_coder_moe_widths_batch8(cuda_device):
    """Qwen3-Coder-30B-A3B widths at batch 8: 128 verify rows route to nearly
    every expert, so the decode takes the dense-routing expert kernels."""
    cfg, gpu, spec = _widths_pair("qwen3_coder_30b_a3b", 8, 96)
    try:
        prompts = [make_prompt("zipf", 6 + 3 * i, cfg.target.vocab, cfg.seed + i) for i in range(8)]
        rep = replay(gpu, spec, cfg, prompts, 2, 3e-2, 0.05)
        print(f"moe batch 8: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
    finally:
        gpu.close()
        torch.cuda.empty_cache()


def test_qwen3_8b_widths_520_token_context(cuda_device):
    """The timed workload's context length: a 520-token Zipf prompt (prefill in
    one chunk through the tensor-core path), two free iterations, then one full
    acceptance and one at k = 5 with the oracle's continuation as drafts."""
    cfg, gpu, spec = _widths_pair("qwen3_8b", 1, 640)
    try:
        prompt = make_prompt("zipf", 520, cfg.target.vocab, cfg.seed)
        rep = replay(gpu, spec, cfg, [prompt], 2, 3e-2, 0.05)
        print(f"520 ctx: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= 3e-2, rep.max_dlogit
        rep2 = replay_forced(gpu, spec, cfg, prompt, (15, 5), 3e-2, 0.05)
        assert rep2.mismatches_outside_ties == 0, rep2
        assert rep2.max_dlogit <= 3e-2, rep2.max_dlogit
    finally:
        gpu.close()
        torch.cuda.empty_cache()


def test_host_wait_timeout_reports_etimeout(cuda_device):
    """timeout_ms = 1 on a pass that takes longer (a 1000-token prefill at the
    Qwen3-8B widths): the host wait gives up with DFLASH_ETIMEOUT while the
    kernels finish on their own; the stream is synchronised before the context
    and its arenas are released."""
    cfg = shrink(get_config("qwen3_8b"), target_layers=2, drafter_layers=1)
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=1100, timeout_ms=1)
    try:
        gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
        with pytest.raises(dfl.DFlashError) as e:
            gpu.prefill(0, make_prompt("zipf", 1000, cfg.target.vocab, 1))
        assert e.value.status == dfl.DFLASH_ETIMEOUT
    finally:
        torch.cuda.synchronize()
        gpu.close()
        torch.cuda.empty_cache()
