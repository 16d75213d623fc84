"""MXFP4 weight streaming on the GPU against the fp64 oracle of the quantised model.

Every projection matrix (and the LM head and the fuse W_fc) is stored as
packed E2M1 codes, one power-of-two exponent per 32 values of a row and one
fp32 scale per row (synthetic.fp4); the kernels stream the 4-bit codes into
block-scaled tensor-core MMAs (the exponents as the weights' scale factors, the
activations as four E4M3 planes with a power-of-two scale per 32 values) and
apply the row scales in the epilogue.  The oracle computes the same quantised
model in fp64, so the same bars hold as for bf16 and FP8 weights: logits within
3e-2, token ids equal outside oracle near-ties (margin < 0.05), integer results
bit for bit.
"""
import pytest
import torch

import block_diffusion_speculative_layers_b200 as dfl
import oracle
from synthetic import get_config, make_prompt, make_weight
from synthetic.configs import shrink
from synthetic.fast import make_weights_host

from parity import build_pair, check_lossless_generate, replay, replay_forced
from test_parity_gpu import tiny_cfg

pytestmark = pytest.mark.gpu

TOL, TIE = 3e-2, 0.05


@pytest.mark.parametrize("case", ["block4", "block16", "wide", "batch3", "chunked"])
def test_fp4_tiny_replay(cuda_device, case):
    kw = dict(dtype="fp4")
    lens, chunk = [30], 0
    if case in ("block16", "wide", "chunked"):
        kw["block"] = 16
    if case == "wide":  # K split across a cluster, several tiles per projection
        kw.update(hidden=2048, nq=16, nkv=4, hd=128, vocab=8192)
    if case == "batch3":
        kw["block"] = 8
        lens = [17, 40, 33]
    if case == "chunked":
        chunk, lens = 16, [45]
    cfg = tiny_cfg(**kw)
    gpu, spec, _ = build_pair(cfg, max_batch=len(lens), max_len=256, prefill_chunk=chunk)
    prompts = [make_prompt("uniform", L, cfg.target.vocab, 80 + i) for i, L in enumerate(lens)]
    rep = replay(gpu, spec, cfg, prompts, 5, TOL, TIE)
    print(f"fp4 {case}: max |dlogit| {rep.max_dlogit:.2e}, near ties {rep.near_ties}/{rep.checked_tokens}")
    assert rep.mismatches_outside_ties == 0, rep
    assert rep.max_dlogit <= TOL


def test_fp4_forced_acceptance_and_lossless_generation(cuda_device):
    cfg = tiny_cfg("fp4", block=16)
    gpu, spec, _ = build_pair(cfg, max_len=160)
    prompt = make_prompt("uniform", 20, cfg.target.vocab, 90)
    rep = replay_forced(gpu, spec, cfg, prompt, (15, 6, 0), TOL, TIE)
    assert rep.mismatches_outside_ties == 0 and rep.max_dlogit <= TOL
    k, st = check_lossless_generate(gpu, spec, cfg, make_prompt("uniform", 25, cfg.target.vocab, 91), 60, TIE)
    assert st.tokens == 59


def test_fp4_qwen3_8b_widths(cuda_device):
    """The Qwen3-8B widths (hidden 4096, FFN 12288, vocab 151936) with MXFP4 weights:
    two target layers and one drafter layer, two iterations."""
    cfg = shrink(get_config("qwen3_8b"), target_layers=2, drafter_layers=1).with_(dtype="fp4")
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=128, keep_logits=True)
    try:
        gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
        spec = oracle.OracleSpec(cfg, make_weights_host(cfg))
        rep = replay(gpu, spec, cfg, [make_prompt("zipf", 24, cfg.target.vocab, cfg.seed)], 2, TOL, TIE)
        print(f"fp4 qwen widths: max |dlogit| {rep.max_dlogit:.2e}, near ties {rep.near_ties}/{rep.checked_tokens}")
        assert rep.mismatches_outside_ties == 0, rep
        assert rep.max_dlogit <= TOL
    finally:
        gpu.close()
        torch.cuda.empty_cache()


def test_fp4_refuses_widths_off_the_128_grid(cuda_device):
    cfg = tiny_cfg("fp4", hidden=192)
    with pytest.raises(dfl.DFlashError):
        dfl.DFlash(cfg, max_batch=1, max_len=64)
