"""The allocation-free greedy-head entry point agrees with the regular path.

dflash_head_argmax_noalloc serves callers that cannot give the library more
device memory when they call it (a serving process whose device memory pool
is fully reserved, or a decode thread that must not call cudaMalloc).  It
recomputes the LM-head argmax of the last pass with its scratch in a static
device array; the ids must equal the ones the regular entry points returned
(dflash_prefill's first token, dflash_draft_block's drafts, and the target
argmax of dflash_verify_commit's rows) on two consecutive iterations.  Ids are
compared exactly, as everywhere else in the parity tests.

Cases: the tiny model (8 vocabulary tiles); a 151936-entry vocabulary (1187
tiles) at the 64-row limit, once with the RMSNorm folded into the head's
projection (the head reads x * g with a per-row scale) and once with a
separate RMSNorm kernel (the head reads the normalised rows); and the error
returns -- more than 64 rows, no pass yet, a pass of another kind last.
"""
from dataclasses import replace

import numpy as np
import pytest

import block_diffusion_speculative_layers_b200 as dfl
from synthetic import get_config, make_prompt, make_weights

pytestmark = pytest.mark.gpu


def _cfg(block, vocab=None):
    base = get_config("tiny")
    cfg = base.with_(dtype="bf16", block_size=block)
    if vocab:
        cfg = cfg.with_(target=replace(cfg.target, vocab=vocab), drafter=replace(cfg.drafter, vocab=vocab))
    return cfg


def _ctx(cfg, max_batch=2, max_len=160):
    ctx = dfl.DFlash(cfg, max_batch=max_batch, max_len=max_len, keep_logits=True)
    ctx.load_weights(make_weights(cfg, device="cuda", random_gains=True))
    return ctx


def _two_iterations(cfg, ctx, n_seq, seqs=None):
    B = cfg.block_size
    seqs = list(range(n_seq)) if seqs is None else seqs
    for seq in range(n_seq):
        first = ctx.prefill(seq, make_prompt("uniform", 20 + seq, cfg.target.vocab, 3 + seq))
        np.testing.assert_array_equal(ctx.head_argmax_noalloc(2), [first])
    for _ in range(2):  # two calls in a row on each pass kind
        drafts = ctx.draft_block(seqs)
        np.testing.assert_array_equal(ctx.head_argmax_noalloc(0), drafts.reshape(-1))
        acc, com, nl = ctx.verify_commit(seqs)
        g = np.argmax(ctx.debug_logits(1, n_seq * B), axis=-1)
        got = ctx.head_argmax_noalloc(1)
        np.testing.assert_array_equal(got, g)
        for i in range(n_seq):
            a = int(acc[i])
            assert list(com[i][:a + 1]) == list(drafts[i][:a]) + [int(got[i * B + a])]


@pytest.mark.parametrize("block", [4, 16])
def test_noalloc_head_matches_regular_entry_points(cuda_device, block):
    cfg = _cfg(block)
    ctx = _ctx(cfg)
    _two_iterations(cfg, ctx, 2)
    ctx.close()


@pytest.mark.parametrize("folded", [True, False])
def test_noalloc_head_full_vocab_64_rows(cuda_device, folded, monkeypatch):
    """151936-entry vocabulary and 4 x 16 = 64 rows (the documented limits of rows;
    1187 of the 2048 vocabulary tiles), with the head's RMSNorm folded into the
    projection or as a separate kernel (DFLASH_FOLDED_NORM=0)."""
    if not folded:
        monkeypatch.setenv("DFLASH_FOLDED_NORM", "0")
    cfg = _cfg(16, vocab=151936)
    ctx = _ctx(cfg, max_batch=4, max_len=96)
    _two_iterations(cfg, ctx, 4)
    ctx.close()


def test_noalloc_head_error_returns(cuda_device):
    cfg = _cfg(16)
    ctx = _ctx(cfg, max_batch=5, max_len=96)

    def status(which):
        with pytest.raises(dfl.DFlashError) as e:
            ctx.head_argmax_noalloc(which)
        return e.value.status

    for which in (0, 1, 2):  # no pass has run yet
        assert status(which) == dfl.DFLASH_ESTATE
    for seq in range(5):
        ctx.prefill(seq, make_prompt("uniform", 12, cfg.target.vocab, seq))
    ctx.head_argmax_noalloc(2)
    ctx.draft_block([0, 1])
    assert status(2) == dfl.DFLASH_ESTATE          # the last pass is a draft
    assert status(1) == dfl.DFLASH_ESTATE
    assert len(ctx.head_argmax_noalloc(0)) == 2 * 15
    ctx.verify_commit([0, 1])
    assert status(0) == dfl.DFLASH_ESTATE          # the last pass is a verify
    ctx.draft_block([0, 1, 2, 3, 4])               # 80 rows: above the 64-row limit
    assert status(0) == dfl.DFLASH_ECAPACITY
    ctx.verify_commit([0, 1, 2, 3, 4])
    assert status(1) == dfl.DFLASH_ECAPACITY
    ctx.decode_iters(5, 1)                         # a decode loop is not a pass of either kind
    assert status(1) == dfl.DFLASH_ESTATE
    ctx.set_draft_mode(dfl.DFLASH_DRAFT_SCRIPT, 2)
    ctx.set_script(0, np.arange(80, dtype=np.int32))
    ctx.draft_block([0])
    assert status(0) == dfl.DFLASH_ESTATE          # script drafts are not the argmax
    ctx.close()
