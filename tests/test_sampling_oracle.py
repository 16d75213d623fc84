"""Pins of the temperature-sampling oracle (oracle/sampling.py).  CPU only.

- Philox4x32-10 against the generator's published known-answer vectors;
- the uniform mapping against its closed-form end points, and the draws
  against U(0, 1) (Kolmogorov-Smirnov);
- Gumbel-max draws against softmax (chi-squared), with a planted sign mistake
  that the same test rejects;
- the acceptance rule: one-hot distributions reduce it to the greedy rule of
  the hand-worked fixture; a toy autoregressive target and drafter give
  committed sequences whose distribution is the target's own closed-form
  product of conditionals (chi-squared), and an off-by-one row mistake
  planted in the inputs is rejected;
- the draft-and-verify and target-only sampling loops on the oracle's model
  become greedy decoding as the temperature vanishes.
"""
from __future__ import annotations

import itertools
import os

import numpy as np
import pytest
from scipy import stats

import oracle
from oracle import sampling as S
from synthetic import make_prompt, make_weights

from test_oracle_pins import tiny

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- Philox and uniforms
def test_philox_known_answer_vectors():
    rows = [l for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip() and l[0] != "#"]
    assert len(rows) == 3
    for l in rows:
        ctr, key, out = ([int(w, 16) for w in part.split()] for part in l.split("|"))
        got = S.philox4x32_10(np.array(ctr, np.uint32), np.array(key, np.uint32))
        assert [int(x) for x in got] == out


def test_uniform_mapping_end_points_are_exact_in_fp32():
    u = S.word_to_uniform(np.array([0, 511, 512, 0xFFFFFFFF], np.uint32))
    assert u[0] == 2.0 ** -24 and u[1] == 2.0 ** -24          # the low 9 bits are dropped
    assert u[2] == 3 * 2.0 ** -24
    assert u[3] == 1.0 - 2.0 ** -24
    assert (u.astype(np.float32).astype(np.float64) == u).all()
    assert ((u > 0) & (u < 1)).all()


def test_draws_are_uniform_and_streams_differ():
    v = S.uniform_vector(2024, 3, 17, S.DRAFT, 200_000)
    assert stats.kstest(v, "uniform").pvalue > 1e-3
    assert ((v > 0) & (v < 1)).all()
    w = S.uniform_vector(2024, 3, 17, S.RESIDUAL, 4096)
    x = S.uniform_vector(2024, 3, 18, S.DRAFT, 4096)
    y = S.uniform_vector(2024, 4, 17, S.DRAFT, 4096)
    z = S.uniform_vector(2025, 3, 17, S.DRAFT, 4096)
    for other in (w, x, y, z):
        assert np.mean(other == v[:4096]) < 1e-3
        assert abs(np.corrcoef(other, v[:4096])[0, 1]) < 0.06
    # all four words of a Philox block are used, in order
    assert len(np.unique(v[:4096])) > 4000
    assert S.uniform_scalar(2024, 3, 17, S.DRAFT) == v[0]


# ---------------------------------------------------------------- Gumbel-max
def _gumbel_counts(z, T, n):
    counts = np.zeros(len(z), np.int64)
    for pos in range(n):
        i, _ = S.gumbel_argmax(np.asarray(z) / T, S.uniform_vector(11, 0, pos, S.TARGET, len(z)))
        counts[i] += 1
    return counts


def test_gumbel_argmax_samples_the_softmax(monkeypatch):
    z = np.array([0.3, -1.1, 0.9, 0.0, -0.4, 1.4])
    T, n = 0.8, 20_000
    p = S.softmax_t(z, T)
    counts = _gumbel_counts(z, T, n)
    assert stats.chisquare(counts, n * p).pvalue > 1e-3
    # a planted sign mistake (the Gumbel minimum instead of the maximum) fails the same test
    monkeypatch.setattr(S, "gumbel", lambda u: np.log(-np.log(np.asarray(u, np.float64))))
    wrong = _gumbel_counts(z, T, n)
    assert stats.chisquare(wrong, n * p).pvalue < 1e-12


def test_gumbel_argmax_excludes_minus_infinity_and_breaks_ties_low():
    u = np.full(4, 0.5)
    assert S.gumbel_argmax(np.array([-np.inf, 1.0, 1.0, -np.inf]), u)[0] == 1
    i, m = S.gumbel_argmax(np.array([-np.inf, -np.inf, 0.0]), np.array([0.9, 0.1, 1e-6]))
    assert i == 2 and m == np.inf


# ---------------------------------------------------------------- the acceptance rule
def _one_hot(ids, V):
    m = np.zeros((len(ids), V))
    m[np.arange(len(ids)), ids] = 1.0
    return m


def test_one_hot_distributions_reduce_to_the_greedy_rule():
    """With P rows one-hot at the target argmax g and Q rows one-hot at the
    drafts, the rule commits d_1 .. d_a and g_a: the hand-worked greedy cases."""
    rows = [l for l in open(os.path.join(GOLDEN, "accept_rule.txt")) if l.strip() and l[0] != "#"]
    V = 16
    for n, l in enumerate(rows):
        B, d, g, a, committed = (part.split() for part in l.split("|"))
        B, a = int(B[0]), int(a[0])
        d, g, committed = [int(x) for x in d], [int(x) for x in g], [int(x) for x in committed]
        o = S.accept_block(_one_hot(g, V), _one_hot(d, V), d, 40, S.Noise(5, n))
        assert o.a == a and d[:o.a] + [o.x] == committed


def test_drafter_equal_to_target_accepts_everything():
    rng = np.random.default_rng(1)
    B, V = 5, 7
    P = S.softmax_t(rng.normal(size=(B, V)), 1.0)
    for seq in range(50):
        o = S.accept_block(P, P[:B - 1], rng.integers(0, V, B - 1), 3, S.Noise(9, seq))
        assert o.a == B - 1 and not o.from_residual


def test_rejected_draft_is_replaced_from_the_positive_part():
    P = np.array([[0.5, 0.5, 0.0, 0.0], [0.25, 0.25, 0.25, 0.25]])
    Q = np.array([[0.0, 0.2, 0.8, 0.0]])
    for seq in range(200):  # d_1 = 2 has P = 0: always rejected; P - Q > 0 only at 0 and 1
        o = S.accept_block(P, Q, [2], 10, S.Noise(3, seq))
        assert o.a == 0 and o.from_residual and o.x in (0, 1)


class ToyLM:
    """A toy autoregressive target and a toy block drafter over a small vocabulary:
    next-token logits drawn once per context from a seeded generator."""

    def __init__(self, V, seed, scale):
        self.V, self.seed, self.scale, self.cache = V, seed, scale, {}

    def logits(self, key):
        if key not in self.cache:
            rng = np.random.default_rng([self.seed, len(key)] + [int(k) for k in key])
            self.cache[key] = rng.normal(scale=self.scale, size=self.V)
        return self.cache[key]


def _toy_generate(target, drafter, prompt, N, B, T, noise, row_shift=0):
    """Draft-and-verify sampling on the toy models (the oracle's loop, with the
    toy models in place of the transformer); row_shift != 0 plants an
    off-by-one mistake in the rows given to the rule."""
    out = []
    anchor, _ = S.sample_target(target.logits(tuple(prompt)), T, len(prompt), noise)
    out.append(anchor)
    while len(out) < N:
        ctx = tuple(prompt) + tuple(out)
        p = len(ctx) - 1
        q_logits = np.stack([drafter.logits(ctx + (drafter.V + i,)) for i in range(1, B)])
        drafts, _ = S.sample_drafts(q_logits, T, p, noise)
        rows = np.stack([target.logits(ctx + tuple(int(x) for x in drafts[:i])) for i in range(B)])
        P = S.softmax_t(rows, T)
        if row_shift:
            P = np.roll(P, row_shift, axis=0)
        o = S.accept_block(P, S.softmax_t(q_logits, T), drafts, p, noise)
        out.extend(int(x) for x in drafts[:o.a])
        out.append(o.x)
    return tuple(out[:N])


def _target_law(target, prompt, N, T):
    law = {}
    for s in itertools.product(range(target.V), repeat=N):
        pr = 1.0
        for j in range(N):
            pr *= S.softmax_t(target.logits(tuple(prompt) + s[:j]), T)[s[j]]
        law[s] = pr
    return law


@pytest.mark.parametrize("row_shift", [0, 1])
def test_draft_and_verify_sampling_keeps_the_target_distribution(row_shift):
    V, N, B, T, runs = 3, 3, 3, 1.0, 12_000
    target, drafter = ToyLM(V, 1, 0.8), ToyLM(V, 2, 0.8)
    prompt = (0, 2)
    law = _target_law(target, prompt, N, T)
    assert abs(sum(law.values()) - 1.0) < 1e-12
    counts = dict.fromkeys(law, 0)
    for r in range(runs):
        counts[_toy_generate(target, drafter, prompt, N, B, T, S.Noise(77, r), row_shift)] += 1
    keys = sorted(law)
    obs = np.array([counts[k] for k in keys])
    exp = np.array([law[k] for k in keys]) * runs
    assert exp.min() > 20
    pv = stats.chisquare(obs, exp).pvalue
    if row_shift == 0:
        assert pv > 1e-3, pv
    else:  # the planted mistake is detected
        assert pv < 1e-10, pv


# ---------------------------------------------------------------- the loops on the oracle's model
def test_sampling_becomes_greedy_as_temperature_vanishes():
    cfg = tiny(block=4)
    spec = oracle.OracleSpec(cfg, make_weights(cfg))
    prompt = make_prompt("uniform", 12, cfg.target.vocab, 6)
    ar = spec.generate_ar(prompt, 20)
    out, acc = spec.generate_spec(prompt, 20)
    s_ar, s_ar_mg = S.generate_ar_sample(spec, prompt, 20, 1e-7, seed=3)
    s_out, s_acc = S.generate_spec_sample(spec, prompt, 20, 1e-7, seed=3)
    np.testing.assert_array_equal(s_ar, ar)
    np.testing.assert_array_equal(s_out, out)
    np.testing.assert_array_equal(s_acc, acc)
    assert (s_ar_mg > 0).all()


def test_sampling_loops_are_deterministic_in_the_seed_and_log_their_decisions():
    cfg = tiny(block=4)
    spec = oracle.OracleSpec(cfg, make_weights(cfg))
    prompt = make_prompt("uniform", 10, cfg.target.vocab, 8)
    seen = []
    a1, acc1 = S.generate_spec_sample(spec, prompt, 12, 0.7, seed=21, log=lambda *x: seen.append(x))
    a2, acc2 = S.generate_spec_sample(spec, prompt, 12, 0.7, seed=21)
    b, _ = S.generate_spec_sample(spec, prompt, 12, 0.7, seed=22)
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(acc1, acc2)
    assert not np.array_equal(a1, b)
    assert len(seen) == len(acc1)
    for (p, drafts, dmg, o), a in zip(seen, acc1):
        assert o.a == a and len(drafts) == cfg.block_size - 1 and len(o.accept_margins) == min(a + 1, cfg.block_size - 1)
    # the first token is the target's sample at the prompt's end, as in target-only sampling
    c, _ = S.generate_ar_sample(spec, prompt, 4, 0.7, seed=21)
    assert a1[0] == c[0]
