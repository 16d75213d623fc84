"""Temperature sampling on the GPU against the oracle's sampling rule.

The GPU and the oracle draw the same Philox4x32-10 numbers, so sampled tokens
are argmaxes of the same perturbed scores and are compared token for token,
teacher-forced on the GPU's commits: drafts, each acceptance decision, and the
token after the accepted drafts (residual draw or bonus).  A decision may
differ only where the oracle's own decision is a near tie at the logits'
bf16 tolerance; those are counted.  The T -> 0 limit must reproduce greedy
decoding exactly, and the draws depend only on (seed, slot, position).
"""
import numpy as np
import pytest

import block_diffusion_speculative_layers_b200 as dfl
import oracle
from oracle import sampling as S
from synthetic import make_prompt, make_weight
from synthetic.fast import make_weights_host

from test_parity_gpu import tiny_cfg

pytestmark = pytest.mark.gpu

LOGIT_TOL = 3e-2  # bf16 logits against the fp64 oracle


def _pair(cfg, max_len=256, **kw):
    gpu = dfl.DFlash(cfg, max_batch=1, max_len=max_len, keep_logits=True, sampling=True, **kw)
    gpu.load_weights_from(lambda n: make_weight(cfg, n, device="cuda"))
    return gpu, oracle.OracleSpec(cfg, make_weights_host(cfg))


def sampled_replay(gpu, spec, cfg, prompt, iters, T, seed):
    """Teacher-forced replay of `iters` sampled iterations of slot 0."""
    B = cfg.block_size
    tie = 2 * LOGIT_TOL / T  # perturbed scores carry the logit error divided by T
    noise = S.Noise(seed, 0)
    n = len(prompt)
    counts = dict(checked=0, ties=0)

    def agree(same, margin):
        counts["checked"] += 1
        if not same:
            assert margin < tie, (margin, tie)
            counts["ties"] += 1

    first = gpu.prefill(0, prompt)
    ss = spec.session(n + (iters + 2) * B + 8)
    _, _, lg = ss.prefill(prompt, want_logits=True)
    o_first, m = S.sample_target(lg, T, n, noise)
    agree(first == o_first, m)
    anchor = first
    for _ in range(iters):
        p = ss.len
        d = gpu.draft_block([0])[0]
        _, _, q = ss.draft(anchor, want_logits=True)
        od, dm = S.sample_drafts(q, T, p, noise)
        for k in range(B - 1):
            agree(d[k] == od[k], dm[k])
        acc, com, nl = gpu.verify_commit([0])
        a = int(acc[0])
        _, _, plog = ss.verify([anchor] + [int(t) for t in d], want_logits=True)
        P, Q = S.softmax_t(plog, T), S.softmax_t(q, T)
        for k in range(1, min(a + 2, B)):
            dk = int(d[k - 1])
            uq, pk = noise.scalar(p + k, S.ACCEPT) * Q[k - 1, dk], P[k - 1, dk]
            rel = abs(uq - pk) / max(uq, pk)
            agree((uq < pk) == (k <= a), rel)
        x = int(com[0][a])
        assert list(com[0][:a]) == [int(t) for t in d[:a]]
        o = S.accept_block(P, Q, d, p, noise)
        if a < B - 1:
            assert P[a, x] - Q[a, x] > -1e-6, "the replacement lies outside max(0, P - Q)"
        if o.a == a:
            agree(x == o.x, o.x_margin)
        assert int(nl[0]) == p + a + 1
        ss.commit(a)
        anchor = x
    return counts


@pytest.mark.parametrize("block,T", [(4, 0.8), (16, 1.0), (8, 0.3)])
def test_sampled_iterations_match_the_oracle(cuda_device, block, T):
    cfg = tiny_cfg(dtype="bf16", block=block)
    gpu, spec = _pair(cfg)
    try:
        gpu.set_sampling(T, seed=1234 + block)
        prompt = make_prompt("uniform", 24, cfg.target.vocab, 3)
        c = sampled_replay(gpu, spec, cfg, prompt, 8, T, 1234 + block)
        print(f"block {block} T {T}: {c['ties']} near ties of {c['checked']} decisions")
        assert c["ties"] <= max(2, c["checked"] // 20)
    finally:
        gpu.close()


def test_sampling_at_vanishing_temperature_is_greedy(cuda_device):
    cfg = tiny_cfg(dtype="bf16", block=4)
    gpu, _ = _pair(cfg)
    try:
        prompt = make_prompt("uniform", 20, cfg.target.vocab, 5)
        greedy, _ = gpu.generate([prompt], 40)
        gpu.set_sampling(1e-6, seed=7)
        sampled, _ = gpu.generate([prompt], 40)
        np.testing.assert_array_equal(sampled[0], greedy[0])
        ar_s, _ = gpu.generate_ar([prompt], 20)
        gpu.set_sampling(0.0)
        ar_g, _ = gpu.generate_ar([prompt], 20)
        np.testing.assert_array_equal(ar_s[0], ar_g[0])
    finally:
        gpu.close()


def test_draws_depend_on_the_seed_only(cuda_device):
    cfg = tiny_cfg(dtype="bf16", block=4)
    gpu, _ = _pair(cfg)
    try:
        prompt = make_prompt("uniform", 16, cfg.target.vocab, 6)
        gpu.set_sampling(0.9, seed=11)
        a, _ = gpu.generate([prompt], 32)
        b, _ = gpu.generate([prompt], 32)
        gpu.set_sampling(0.9, seed=12)
        c, _ = gpu.generate([prompt], 32)
        np.testing.assert_array_equal(a[0], b[0])
        assert not np.array_equal(a[0], c[0])
    finally:
        gpu.close()


def test_sampling_arguments_are_checked(cuda_device):
    cfg = tiny_cfg(dtype="bf16", block=4)
    plain = dfl.DFlash(cfg, max_batch=1, max_len=64)
    try:
        with pytest.raises(dfl.DFlashError) as e:
            plain.set_sampling(0.7, 1)
        assert e.value.status == dfl.DFLASH_ESTATE
        plain.set_sampling(0.0, 1)  # greedy is always allowed
    finally:
        plain.close()
    gpu, _ = _pair(cfg, max_len=64)
    try:
        for bad in (-1.0, float("nan"), float("inf")):
            with pytest.raises(dfl.DFlashError) as e:
                gpu.set_sampling(bad, 1)
            assert e.value.status == dfl.DFLASH_EINVAL
        gpu.set_sampling(0.5, 1)
        with pytest.raises(dfl.DFlashError) as e:
            gpu.set_draft_mode(dfl.DFLASH_DRAFT_SCRIPT, 2)
        assert e.value.status == dfl.DFLASH_ESTATE
    finally:
        gpu.close()
