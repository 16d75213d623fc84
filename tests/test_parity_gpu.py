"""GPU parity of the CUDA path against the fp64 oracle (teacher-forced replay).

Tolerances: fp32 models, logits within 1e-4 and token ties below a 1e-3 margin;
bf16 models, logits within 3e-2 and ties below a 0.05 margin (bf16 weights and
GEMM inputs against fp64 arithmetic).  Integer results (accept lengths,
committed tokens, new lengths) are always compared bit for bit.
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import pytest
import torch

import block_diffusion_speculative_layers_b200 as dfl
from synthetic import get_config, make_prompt
from synthetic.configs import ModelDims

import oracle
from synthetic import make_weights
from synthetic.fast import make_weights_host
from parity import build_pair, replay, replay_forced, check_lossless_generate, accept_rule

pytestmark = pytest.mark.gpu

TOL = {"fp32": (1e-4, 1e-3), "bf16": (3e-2, 0.05)}


def tiny_cfg(dtype="fp32", block=4, moe=False, t_layers=2, d_layers=1, nq=4, nkv=2, hd=64, hidden=256,
             vocab=1024, taps=(0, 1), expert_ffn=64, qk_norm=False, rope_scaling=None):
    base = get_config("tiny")
    ffn = 3 * hidden
    fid = dict(qk_norm=qk_norm)
    if rope_scaling is not None:
        fid["rope_scaling"] = rope_scaling
    t = replace(base.target, n_layers=t_layers, n_q_heads=nq, n_kv_heads=nkv, head_dim=hd, hidden=hidden,
                vocab=vocab, ffn=ffn, **fid)
    if moe:
        t = replace(t, n_experts=8, top_k=2, expert_ffn=expert_ffn)
    d = replace(base.drafter, n_layers=d_layers, n_q_heads=nq, n_kv_heads=nkv, head_dim=hd, hidden=hidden,
                vocab=vocab, ffn=ffn, **fid)
    return base.with_(target=t, drafter=d, block_size=block, tap_layers=taps, dtype=dtype)


def _finish(rep, tol, strict=True):
    assert rep.max_dlogit <= tol, rep.max_dlogit
    if strict:
        assert rep.mismatches_outside_ties == 0, rep


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_tiny_replay(cuda_device, dtype):
    cfg = tiny_cfg(dtype)
    tol, tie = TOL[dtype]
    gpu, spec, _ = build_pair(cfg, max_len=256)
    prompt = make_prompt("uniform", 32, cfg.target.vocab, 0)
    rep = replay(gpu, spec, cfg, [prompt], 12, tol, tie)
    _finish(rep, tol)


def test_config1_generate_is_lossless(cuda_device):
    """Tiny fp32 configuration: 32-token prompt, 64 generated tokens."""
    cfg = get_config("tiny")
    gpu, spec, _ = build_pair(cfg, max_len=128, random_gains=False)
    prompt = make_prompt(cfg.prompt_kind, cfg.prompt_len, cfg.target.vocab, cfg.seed)
    k, st = check_lossless_generate(gpu, spec, cfg, prompt, cfg.max_new, TOL["fp32"][1])
    assert st.tokens == cfg.max_new - 1
    assert 1.0 <= st.mean_tau <= cfg.block_size


@pytest.mark.parametrize("case", ["block16", "moe", "moe_bucketed", "moe_stream", "mha_hd128", "chunked_prefill",
                                  "batch3", "wide", "wide_batch2"])
def test_bf16_variants_replay(cuda_device, case, monkeypatch):
    kw = dict(dtype="bf16")
    if case == "moe_stream":  # the CUDA-core weight-streaming expert kernels instead of the grouped projections
        monkeypatch.setenv("DFLASH_MOE_STREAM", "1")
    prompts_n, lens, chunk = 1, [40], 0
    if case == "block16":
        kw.update(block=16)
    if case == "moe":
        kw.update(moe=True)                   # expert FFN 64: CUDA-core expert kernel
    if case in ("moe_bucketed", "moe_stream"):
        kw.update(moe=True, expert_ffn=256)   # bucketed experts (hidden and expert FFN multiples of 256)
    if case == "mha_hd128":
        kw.update(nq=2, nkv=2, hd=128)
    if case == "chunked_prefill":
        chunk = 16
        lens = [45]
    if case == "batch3":
        kw.update(block=8)
        lens = [17, 40, 33]
    if case in ("wide", "wide_batch2"):
        # wide enough that projections split K across CTAs (16-48 tiles per projection)
        kw.update(block=16, hidden=2048, nq=16, nkv=4, hd=128, vocab=8192)
        if case == "wide_batch2":
            lens = [30, 21]
    cfg = tiny_cfg(**kw)
    tol, tie = TOL["bf16"]
    gpu, spec, _ = build_pair(cfg, max_batch=len(lens), max_len=256, prefill_chunk=chunk)
    prompts = [make_prompt("uniform", L, cfg.target.vocab, 10 + i) for i, L in enumerate(lens)]
    rep = replay(gpu, spec, cfg, prompts, 6, tol, tie)
    _finish(rep, tol)


def test_script_mode_forces_accept_length(cuda_device):
    cfg = tiny_cfg("fp32", block=8)
    gpu, spec, _ = build_pair(cfg, max_len=256)
    prompt = make_prompt("uniform", 20, cfg.target.vocab, 3)
    ar, _ = gpu.generate_ar([prompt], 120)
    for tau in (1, 3, 8):
        gpu.set_script(0, ar[0])
        gpu.set_draft_mode(dfl.DFLASH_DRAFT_SCRIPT, tau)
        out, st = gpu.generate([prompt], 100)
        np.testing.assert_array_equal(out[0], ar[0][:100])
        hist = np.array(st.accept_hist[:cfg.block_size])
        # every iteration commits exactly tau tokens (the last one may be truncated)
        assert hist[tau - 1] >= hist.sum() - 1, (tau, hist)
    gpu.set_draft_mode(dfl.DFLASH_DRAFT_MODEL, 1)


def test_gpu_spec_equals_gpu_ar(cuda_device):
    cfg = tiny_cfg("bf16", block=16)
    gpu, spec, _ = build_pair(cfg, max_len=256)
    prompt = make_prompt("uniform", 24, cfg.target.vocab, 5)
    ar, _ = gpu.generate_ar([prompt], 80)
    out, st = gpu.generate([prompt], 80)
    div = np.nonzero(out[0] != ar[0])[0]
    if len(div):
        # a divergence may only come from a near-tie of the target
        _, margins = spec.generate_ar(prompt, 80, with_margins=True)
        assert margins[div[0]] < TOL["bf16"][1]


def test_errors_are_reported(cuda_device):
    cfg = tiny_cfg("fp32")
    gpu, spec, _ = build_pair(cfg, max_batch=2, max_len=64)
    prompt = make_prompt("uniform", 10, cfg.target.vocab, 1)
    with pytest.raises(dfl.DFlashError) as e:
        gpu.draft_block([0])                         # slot not prefilled
    assert e.value.status == dfl.DFLASH_ESTATE if hasattr(dfl, "DFLASH_ESTATE") else 2
    gpu.prefill(0, prompt)
    with pytest.raises(dfl.DFlashError) as e:
        gpu.verify_commit([0])                       # no preceding draft
    assert e.value.status == 2
    with pytest.raises(dfl.DFlashError) as e:
        gpu.prefill(1, np.zeros(62, np.int32))       # prompt + block > max_len
    assert e.value.status == 3
    with pytest.raises(dfl.DFlashError) as e:
        gpu.prefill(5, prompt)                       # slot out of range
    assert e.value.status == 1
    with pytest.raises(dfl.DFlashError) as e:
        gpu.prefill(1, [cfg.target.vocab])           # id out of vocab
    assert e.value.status == 1
    # the context stays usable after argument errors
    gpu.draft_block([0])
    acc, com, nl = gpu.verify_commit([0])
    assert 0 <= acc[0] <= cfg.block_size - 1
    # run until capacity: each iteration commits >= 1 token, so ECAPACITY must come
    with pytest.raises(dfl.DFlashError) as e:
        for _ in range(64):
            gpu.draft_block([0])
            gpu.verify_commit([0])
    assert e.value.status == 3


def test_kv_rollback_matches_oracle(cuda_device):
    """After iterations with rejections, the committed target KV and the drafter
    context K/V equal the oracle's at every valid position (stale slots beyond
    the committed length are never read, so they are not compared)."""
    cfg = tiny_cfg("fp32", block=4)
    gpu, spec, _ = build_pair(cfg, max_len=128)
    prompt = make_prompt("uniform", 12, cfg.target.vocab, 7)
    rep = replay(gpu, spec, cfg, [prompt], 6, *TOL["fp32"])
    ss = rep.sessions[0]
    L, anchor, n_out = gpu.seq_state(0)
    assert L == ss.len
    for layer in range(cfg.target.n_layers):
        k, v = gpu.debug_kv(0, layer, 0, 0, L)
        for t in range(L):
            ko, vo = ss.target_kv(layer, t)
            np.testing.assert_allclose(k[t], ko, rtol=0, atol=1e-4)
            np.testing.assert_allclose(v[t], vo, rtol=0, atol=1e-4)
    # drafter context: positions injected so far (the last verify's rows are
    # injected by the next draft, so run one more draft before comparing)
    gpu.draft_block([0])
    ss.draft(anchor)
    for j in range(cfg.drafter.n_layers):
        k, v = gpu.debug_kv(1, j, 0, 0, L)
        for t in range(L):
            ko, vo = ss.ctx_kv(j, t)
            np.testing.assert_allclose(k[t], ko, rtol=0, atol=1e-4)
            np.testing.assert_allclose(v[t], vo, rtol=0, atol=1e-4)


@pytest.mark.parametrize("mode", ["fast", "unfolded", "counters"])
def test_alternative_execution_modes(cuda_device, mode, monkeypatch):
    """The opt-in execution modes compute the same decode step: single-plane bf16
    activations (DFLASH_BF16_FAST, looser logits), separate RMSNorm kernels
    instead of norms folded into the projections, and device completion
    counters between the kernels of a pass."""
    cfg = tiny_cfg(dtype="bf16", block=16, hidden=2048, nq=16, nkv=4, hd=128, vocab=8192)
    tol, tie = TOL["bf16"]
    act = "split"
    if mode == "fast":
        act, tol = "fast", 0.15   # one plane: plain bf16 rounding of GEMM inputs, q and K/V
    if mode == "unfolded":
        monkeypatch.setenv("DFLASH_FOLDED_NORM", "0")
    if mode == "counters":
        monkeypatch.setenv("DFLASH_DEP_COUNTERS", "1")
    w_cpu = make_weights_host(cfg, random_gains=True)
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=256, keep_logits=True, bf16_act=act)
    gpu.load_weights(make_weights(cfg, device="cuda", random_gains=True))
    spec = oracle.OracleSpec(cfg, w_cpu)
    prompt = make_prompt("uniform", 30, cfg.target.vocab, 12)
    rep = replay(gpu, spec, cfg, [prompt], 4, tol, tie)
    print(f"{mode}: max |dlogit| {rep.max_dlogit:.4f}, near ties {rep.near_ties}/{rep.checked_tokens}")
    _finish(rep, tol, strict=(mode != "fast"))
    gpu.close()


@pytest.mark.parametrize("block", [1, 2])
def test_degenerate_block_sizes(cuda_device, block):
    """B = 1: no drafts, every iteration commits the target's own token; B = 2:
    a single draft per block.  Both stay lossless."""
    cfg = tiny_cfg("bf16", block=block)
    tol, tie = TOL["bf16"]
    gpu, spec, _ = build_pair(cfg, max_len=128)
    prompt = make_prompt("uniform", 24, cfg.target.vocab, 5)
    rep = replay(gpu, spec, cfg, [prompt], 6, tol, tie)
    _finish(rep, tol)
    if block == 1:
        assert all(a == 0 for a in rep.accepts)
    k, st = check_lossless_generate(gpu, spec, cfg, prompt, 20, tie)
    assert st.tokens == 19


def test_one_token_prompt_and_short_generations(cuda_device):
    """A one-token prompt, max_new = 1 (the prefill's token only) and max_new = 2."""
    cfg = tiny_cfg("bf16", block=4)
    tol, tie = TOL["bf16"]
    gpu, spec, _ = build_pair(cfg, max_len=64)
    prompt = make_prompt("uniform", 1, cfg.target.vocab, 8)
    rep = replay(gpu, spec, cfg, [prompt], 3, tol, tie)
    _finish(rep, tol)
    for max_new in (1, 2):
        k, st = check_lossless_generate(gpu, spec, cfg, prompt, max_new, tie)
        assert st.tokens == max_new - 1  # the first token comes from the prefill


def test_batch16_block16_uses_wide_row_tiles(cuda_device):
    """16 sequences x 16 rows = 256 verify rows: the large-row-tile decode path of
    the batch sweep, with ragged prompts."""
    cfg = tiny_cfg("bf16", block=16)
    tol, tie = TOL["bf16"]
    gpu, spec, _ = build_pair(cfg, max_batch=16, max_len=128)
    lens = [5 + 3 * i for i in range(16)]
    prompts = [make_prompt("uniform", L, cfg.target.vocab, 40 + i) for i, L in enumerate(lens)]
    rep = replay(gpu, spec, cfg, prompts, 2, tol, tie)
    _finish(rep, tol)


@pytest.mark.parametrize("dtype,block,cuts", [("fp32", 4, (3, 1, 0, 3)), ("bf16", 4, (3, 2, 0)),
                                              ("bf16", 16, (15, 7, 3, 0))])
def test_forced_accept_lengths_against_oracle(cuda_device, dtype, block, cuts):
    """Caller drafts = the oracle's greedy continuation, wrong after k drafts:
    the verify accepts exactly k (k = B-1: the whole block), commits the
    oracle's tokens, and the target / drafter-context K/V of the committed
    positions equal the oracle's."""
    cfg = tiny_cfg(dtype, block=block)
    tol, tie = TOL[dtype]
    gpu, spec, _ = build_pair(cfg, max_len=128)
    prompt = make_prompt("uniform", 14, cfg.target.vocab, 21)
    rep = replay_forced(gpu, spec, cfg, prompt, cuts, tol, tie, kv_tol=1e-4 if dtype == "fp32" else 1e-2)
    _finish(rep, tol)
    assert rep.accepts[0] == cuts[0] or rep.near_ties > 0


def test_nonfinite_logits_report_enumeric(cuda_device):
    """One NaN in the LM head makes one logit of every row non-finite: the
    synchronising calls return DFLASH_ENUMERIC from the device status word."""
    cfg = tiny_cfg("bf16", block=4)
    gpu, spec, _ = build_pair(cfg, max_len=96)
    gpu.weight_view("lm_head")[7, 3] = float("nan")
    torch.cuda.synchronize()
    prompt = make_prompt("uniform", 10, cfg.target.vocab, 2)
    with pytest.raises(dfl.DFlashError) as e:
        gpu.generate([prompt], 12)
    assert e.value.status == dfl.DFLASH_ENUMERIC
    gpu.reset_stats()
    with pytest.raises(dfl.DFlashError) as e:
        gpu.prefill(0, prompt)
    assert e.value.status == dfl.DFLASH_ENUMERIC
    with pytest.raises(dfl.DFlashError) as e:
        gpu.draft_block([0])
    assert e.value.status == dfl.DFLASH_ENUMERIC
    with pytest.raises(dfl.DFlashError) as e:
        gpu.verify_commit([0])
    assert e.value.status == dfl.DFLASH_ENUMERIC


@pytest.mark.parametrize("dtype,toggle", [("fp32", "qk_norm"), ("bf16", "qk_norm"), ("fp32", "rope_scaled"),
                                          ("bf16", "rope_scaled"), ("bf16", "both_hd128")])
def test_fidelity_toggles_replay(cuda_device, dtype, toggle):
    """Fidelity toggles of real checkpoints (not on the pages): Qwen3 QK-norm
    (per-head RMSNorm of q and k before RoPE, context keys included) and the
    Llama 3.1 RoPE frequency rescaling, with prompts long enough that all three
    wavelength bands rotate; bf16 cases take the tensor-core epilogue (head_dim
    64: two heads per 128-row tile; 128: one), fp32 the CUDA-core one."""
    from test_oracle_pins import TINY_ROPE_SCALING
    kw = dict(block=8)
    if toggle in ("qk_norm", "both_hd128"):
        kw["qk_norm"] = True
    if toggle in ("rope_scaled", "both_hd128"):
        kw["rope_scaling"] = TINY_ROPE_SCALING
    if toggle == "both_hd128":
        kw.update(block=16, hidden=512, nq=4, nkv=2, hd=128)
    cfg = tiny_cfg(dtype, **kw)
    tol, tie = TOL[dtype]
    gpu, spec, _ = build_pair(cfg, max_batch=2, max_len=400)
    prompts = [make_prompt("uniform", 300, cfg.target.vocab, 31), make_prompt("uniform", 45, cfg.target.vocab, 32)]
    rep = replay(gpu, spec, cfg, prompts, 4, tol, tie)
    print(f"{toggle} {dtype}: max |dlogit| {rep.max_dlogit:.2e}, near ties {rep.near_ties}/{rep.checked_tokens}")
    _finish(rep, tol)


@pytest.mark.parametrize("block", [32, 24])
def test_blocks_above_16_rows(cuda_device, block):
    """Blocks of 32 and 24 positions (31 / 23 drafts): the attention tiles split
    each block into 16- (or 12-) row tiles of one sequence; replay, forced full
    and partial acceptance, and lossless generation against the oracle."""
    cfg = tiny_cfg("bf16", block=block)
    tol, tie = TOL["bf16"]
    gpu, spec, _ = build_pair(cfg, max_batch=2, max_len=256)
    prompts = [make_prompt("uniform", 20, cfg.target.vocab, 50), make_prompt("uniform", 33, cfg.target.vocab, 51)]
    rep = replay(gpu, spec, cfg, prompts, 3, tol, tie)
    _finish(rep, tol)
    rep2 = replay_forced(gpu, spec, cfg, make_prompt("uniform", 17, cfg.target.vocab, 52), (block - 1, 9, 0), tol, tie,
                         seq=1)
    _finish(rep2, tol)
    k, st = check_lossless_generate(gpu, spec, cfg, prompts[0], 60, tie)
    assert st.tokens == 59
