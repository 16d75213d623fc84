"""The allocation-free greedy-head entry point agrees with the regular path.

dflash_head_argmax_noalloc serves callers that cannot give the library more
device memory when they call it (a serving process whose device memory pool
is fully reserved, or a decode thread that must not call cudaMalloc).  It
recomputes the LM-head argmax of the last pass with its scratch in a static
device array; the ids must equal the ones the regular entry points returned
(dflash_prefill's first token, dflash_draft_block's drafts, and the target
argmax of dflash_verify_commit's rows) on two consecutive iterations.  Ids are
compared exactly, as everywhere else in the parity tests.
"""
from dataclasses import replace

import numpy as np
import pytest

import block_diffusion_speculative_layers_b200 as dfl
from synthetic import get_config, make_prompt, make_weights

pytestmark = pytest.mark.gpu


def _ctx(block):
    base = get_config("tiny")
    cfg = base.with_(dtype="bf16", block_size=block)
    ctx = dfl.DFlash(cfg, max_batch=2, max_len=160, keep_logits=True)
    ctx.load_weights(make_weights(cfg, device="cuda", random_gains=True))
    return cfg, ctx


@pytest.mark.parametrize("block", [4, 16])
def test_noalloc_head_matches_regular_entry_points(cuda_device, block):
    cfg, ctx = _ctx(block)
    B = cfg.block_size
    for seq, seed in ((0, 3), (1, 4)):
        first = ctx.prefill(seq, make_prompt("uniform", 20 + seq, cfg.target.vocab, seed))
        np.testing.assert_array_equal(ctx.head_argmax_noalloc(2), [first])
    for _ in range(2):  # two calls in a row on each pass kind
        drafts = ctx.draft_block([0, 1])
        np.testing.assert_array_equal(ctx.head_argmax_noalloc(0), drafts.reshape(-1))
        acc, com, nl = ctx.verify_commit([0, 1])
        g = np.argmax(ctx.debug_logits(1, 2 * B), axis=-1)
        got = ctx.head_argmax_noalloc(1)
        np.testing.assert_array_equal(got, g)
        for i in range(2):
            a = int(acc[i])
            assert list(com[i][:a + 1]) == list(drafts[i][:a]) + [int(got[i * B + a])]
