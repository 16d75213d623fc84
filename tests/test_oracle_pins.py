"""Pins of the fp64 oracle against things other than itself.

Closed forms, hand-worked fixtures (tests/golden/), library routines (numpy,
scipy) and an independent dense-matrix restatement of the model
(tests/dense_ref.py).  CPU only.
"""
from __future__ import annotations

import math
import os
from dataclasses import replace

import numpy as np
import pytest
import torch
from scipy.special import softmax as sp_softmax

import oracle
from oracle import api as orc
from synthetic import get_config, make_weights, make_prompt
from synthetic.configs import ModelDims

import dense_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# Llama 3.1-style RoPE rescaling scaled to the tiny model (theta 1e4, head_dim 64):
# pairs 0-8 keep their frequency, 9-12 are mixed, 13-31 are divided by 8
TINY_ROPE_SCALING = (8.0, 1.0, 4.0, 256.0)


def tiny(dtype="fp32", block=4, nq=4, nkv=2, moe=False, taps=(0, 1), t_layers=2, d_layers=1,
         vocab=1024, qk_norm=False, rope_scaling=None):
    base = get_config("tiny")
    fid = dict(qk_norm=qk_norm)
    if rope_scaling:
        fid["rope_scaling"] = rope_scaling
    t = replace(base.target, n_layers=t_layers, n_q_heads=nq, n_kv_heads=nkv, vocab=vocab, **fid)
    if moe:
        t = replace(t, n_experts=8, top_k=2, expert_ffn=64)
    d = replace(base.drafter, n_layers=d_layers, n_q_heads=nq, n_kv_heads=nkv, vocab=vocab, **fid)
    return base.with_(target=t, drafter=d, block_size=block, tap_layers=taps, dtype=dtype)


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_row_closed_form():
    for c in (3.0, -0.25):
        x = np.full(64, c)
        y = orc.rmsnorm(x, np.ones(64, np.float32), 1e-6)
        np.testing.assert_allclose(y, np.full(64, c / math.sqrt(c * c + 1e-6)), rtol=1e-14)


def test_rmsnorm_gain_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.normal(size=96)
    g = rng.normal(size=96).astype(np.float32)
    y1 = orc.rmsnorm(x, g, 0.0)
    y2 = orc.rmsnorm(7.5 * x, g, 0.0)
    np.testing.assert_allclose(y1, y2, rtol=1e-13)
    # unit RMS before the gain
    y0 = orc.rmsnorm(x, np.ones(96, np.float32), 0.0)
    assert abs(np.sqrt((y0 ** 2).mean()) - 1.0) < 1e-13
    np.testing.assert_allclose(y1, y0 * g.astype(np.float64), rtol=1e-13)


# ---------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    v = np.random.default_rng(1).normal(size=128)
    np.testing.assert_array_equal(orc.rope(v, 0, 1e6), v)


def test_rope_closed_form_hd4():
    # hd=4, theta=1e4: pairs (0,2) at frequency 1 and (1,3) at frequency 1e4^(-1/2)=0.01
    v = np.array([1.0, 2.0, 3.0, 4.0])
    for pos in (1, 2, 37):
        a0, a1 = pos * 1.0, pos * 0.01
        want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
                3 * math.cos(a0) + 1 * math.sin(a0), 4 * math.cos(a1) + 2 * math.sin(a1)]
        np.testing.assert_allclose(orc.rope(v, pos, 1e4), want, rtol=1e-13, atol=1e-14)


def test_rope_preserves_norm_and_is_relative():
    rng = np.random.default_rng(2)
    q, k = rng.normal(size=64), rng.normal(size=64)
    for m, n, s in ((5, 3, 11), (100, 0, 4000), (7, 7, 1)):
        d1 = orc.rope(q, m, 1e4) @ orc.rope(k, n, 1e4)
        d2 = orc.rope(q, m + s, 1e4) @ orc.rope(k, n + s, 1e4)
        assert abs(d1 - d2) < 1e-10 * max(1.0, abs(d1))
        assert abs(np.linalg.norm(orc.rope(q, m, 1e4)) - np.linalg.norm(q)) < 1e-12


# ---------------------------------------------------------------- matmul
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,K,R", [(5, 3, 1), (33, 67, 4), (128, 256, 16)])
def test_matmul_vs_numpy(dtype, N, K, R):
    g = torch.Generator().manual_seed(N * 1000 + K)
    W = (torch.randn(N, K, generator=g) * 0.5).to(dtype)
    X = np.random.default_rng(K).normal(size=(R, K))
    Y = orc.matmul(W, X)
    want = X @ W.to(torch.float64).numpy().T
    np.testing.assert_allclose(Y, want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- attention
def _load_attention_golden():
    q, ks, vs, out, hd = None, [], [], None, None
    with open(os.path.join(GOLDEN, "attention_worked.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            tag, *vals = line.split()
            vals = [float(x) for x in vals]
            if tag == "hd":
                hd = int(vals[0])
            elif tag == "q":
                q = vals
            elif tag == "k":
                ks.append(vals)
            elif tag == "v":
                vs.append(vals)
            elif tag == "out":
                out = vals
    return hd, np.array(q), np.array(ks), np.array(vs), np.array(out)


def test_attention_hand_worked_golden():
    hd, q, ks, vs, out = _load_attention_golden()
    np.testing.assert_allclose(orc.attend(q, ks, vs), out, rtol=1e-14, atol=1e-14)


def test_attention_special_cases():
    rng = np.random.default_rng(3)
    hd = 16
    v = rng.normal(size=(1, hd))
    np.testing.assert_allclose(orc.attend(rng.normal(size=hd), rng.normal(size=(1, hd)), v), v[0], rtol=1e-15)
    # equal keys -> uniform weights -> mean of values
    k = np.tile(rng.normal(size=hd), (9, 1))
    vv = rng.normal(size=(9, hd))
    np.testing.assert_allclose(orc.attend(rng.normal(size=hd), k, vv), vv.mean(0), rtol=1e-12, atol=1e-14)
    # zero query -> uniform too
    np.testing.assert_allclose(orc.attend(np.zeros(hd), rng.normal(size=(9, hd)), vv), vv.mean(0), rtol=1e-12, atol=1e-14)


def test_attention_vs_scipy_and_permutation():
    rng = np.random.default_rng(4)
    hd, n = 64, 37
    q, k, v = rng.normal(size=hd), rng.normal(size=(n, hd)), rng.normal(size=(n, hd))
    want = sp_softmax(k @ q / math.sqrt(hd)) @ v
    np.testing.assert_allclose(orc.attend(q, k, v), want, rtol=1e-12, atol=1e-13)
    perm = rng.permutation(n)
    np.testing.assert_allclose(orc.attend(q, k[perm], v[perm]), want, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- argmax / accept
def test_argmax_ties_lowest_index_and_margin():
    i, m = orc.argmax([1.0, 3.0, 2.0, 3.0])
    assert i == 1 and m == 0.0
    i, m = orc.argmax([0.5, -1.0, 0.25])
    assert i == 0 and m == 0.25


def _load_accept_golden():
    rows = []
    with open(os.path.join(GOLDEN, "accept_rule.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            B, d, g, a, c = [s.strip() for s in line.split("|")]
            rows.append((int(B), [int(x) for x in d.split()], [int(x) for x in g.split()], int(a),
                         [int(x) for x in c.split()]))
    return rows


def test_accept_hand_derived_golden():
    for B, d, g, a, committed in _load_accept_golden():
        got = orc.accept(d if d else [0], g, B)
        assert got == a, (B, d, g)
        assert (d[:got] + [g[got]]) == committed


def test_accept_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(500):
        B = int(rng.integers(1, 17))
        g = rng.integers(0, 3, size=B)
        d = rng.integers(0, 3, size=max(1, B - 1))
        # largest k such that every prefix of length <= k matches
        ok = [k for k in range(B) if all(d[i] == g[i] for i in range(k))]
        a = orc.accept(d, g, B)
        assert a == max(ok)
        assert 0 <= a <= B - 1


# ---------------------------------------------------------------- FFN / MoE / fuse
def test_dense_ffn_vs_numpy():
    cfg = tiny()
    w = make_weights(cfg, random_gains=True)
    spec = oracle.OracleSpec(cfg, w)
    x = np.random.default_rng(6).normal(size=cfg.target.hidden)
    gu = w["target.L1.w_gate_up"].double().numpy() @ x
    F = cfg.target.ffn
    want = w["target.L1.w_down"].double().numpy() @ ((gu[:F] / (1 + np.exp(-gu[:F]))) * gu[F:])
    np.testing.assert_allclose(spec.ffn("target", 1, x), want, rtol=1e-12, atol=1e-14)


def test_moe_uniform_router_all_experts_is_mean():
    cfg = tiny(moe=True)
    t = replace(cfg.target, top_k=cfg.target.n_experts)
    cfg = cfg.with_(target=t)
    w = make_weights(cfg)
    w["target.L0.w_router"] = torch.zeros_like(w["target.L0.w_router"])
    spec = oracle.OracleSpec(cfg, w)
    x = np.random.default_rng(7).normal(size=cfg.target.hidden)
    Fe = t.expert_ffn
    outs = []
    for e in range(t.n_experts):
        gu = w["target.L0.we_gate_up"][e].double().numpy() @ x
        outs.append(w["target.L0.we_down"][e].double().numpy() @ ((gu[:Fe] / (1 + np.exp(-gu[:Fe]))) * gu[Fe:]))
    np.testing.assert_allclose(spec.ffn("target", 0, x), np.mean(outs, 0), rtol=1e-11, atol=1e-14)


def test_moe_single_expert_equals_dense():
    cfg_m = tiny(moe=True)
    t = replace(cfg_m.target, n_experts=1, top_k=1, expert_ffn=cfg_m.target.ffn)
    cfg_m = cfg_m.with_(target=t)
    wm = make_weights(cfg_m)
    cfg_d = tiny()
    wd = make_weights(cfg_d)
    wd["target.L0.w_gate_up"] = wm["target.L0.we_gate_up"][0].clone()
    wd["target.L0.w_down"] = wm["target.L0.we_down"][0].clone()
    x = np.random.default_rng(8).normal(size=cfg_m.target.hidden)
    a = oracle.OracleSpec(cfg_m, wm).ffn("target", 0, x)
    b = oracle.OracleSpec(cfg_d, wd).ffn("target", 0, x)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_moe_vs_brute_force():
    cfg = tiny(moe=True)
    w = make_weights(cfg)
    spec = oracle.OracleSpec(cfg, w)
    rng = np.random.default_rng(9)
    for _ in range(4):
        x = rng.normal(size=cfg.target.hidden)
        want = dense_ref._moe(cfg.target, w, "target.L1.", x[None])[0]
        np.testing.assert_allclose(spec.ffn("target", 1, x), want, rtol=1e-11, atol=1e-14)


def test_fuse_vs_numpy():
    cfg = tiny()
    w = make_weights(cfg, random_gains=True)
    spec = oracle.OracleSpec(cfg, w)
    taps = np.random.default_rng(10).normal(size=(cfg.n_taps, cfg.target.hidden))
    u = w["fuse.w_fc"].double().numpy() @ taps.reshape(-1)
    want = dense_ref.rms(u, w["fuse.norm"].double().numpy(), cfg.drafter.rms_eps)
    np.testing.assert_allclose(spec.fuse(taps), want, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- whole model
CASES = {
    "fp32": dict(),
    "bf16": dict(dtype="bf16"),
    "moe": dict(moe=True),
    "mha": dict(nq=4, nkv=4),
    "block16": dict(block=16),
    "qk_norm": dict(qk_norm=True),
    "rope_scaled": dict(rope_scaling=TINY_ROPE_SCALING),
}


@pytest.mark.parametrize("case", list(CASES))
def test_target_matches_dense_reference(case):
    cfg = tiny(**CASES[case])
    w = make_weights(cfg, random_gains=True)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 12, cfg.target.vocab, 1)
    out = spec.generate_ar(prompt, 6)
    # independent: recompute the whole prefix every step in matrix form
    toks = list(prompt)
    for i in range(6):
        logits, _ = dense_ref.target_forward(cfg, w, toks)
        nxt = int(np.argmax(logits[-1]))
        assert nxt == out[i], (case, i)
        toks.append(nxt)
    # and the logits of an oracle verify block
    ss = spec.session(64)
    anchor, _, lg0 = ss.prefill(prompt, want_logits=True)
    ref_logits, _ = dense_ref.target_forward(cfg, w, list(prompt))
    np.testing.assert_allclose(lg0, ref_logits[-1], rtol=1e-9, atol=1e-9)
    block = [anchor] + list(range(1, cfg.block_size))
    g, _, lg = ss.verify(block, want_logits=True)
    ref_logits, _ = dense_ref.target_forward(cfg, w, list(prompt) + block)
    np.testing.assert_allclose(lg, ref_logits[len(prompt):], rtol=1e-9, atol=1e-9)


def test_gqa_equals_mha_with_repeated_kv_heads():
    cfg = tiny(nq=4, nkv=2)
    w = make_weights(cfg)
    cfg_m = tiny(nq=4, nkv=4)
    wm = {k: v.clone() for k, v in w.items()}
    d = cfg.target
    hd, qd, kd = d.head_dim, d.q_dim, d.kv_dim
    for l in range(d.n_layers):
        W = w[f"target.L{l}.wqkv"]
        k = W[qd:qd + kd].view(d.n_kv_heads, hd, -1).repeat_interleave(2, dim=0).reshape(-1, W.shape[1])
        v = W[qd + kd:].view(d.n_kv_heads, hd, -1).repeat_interleave(2, dim=0).reshape(-1, W.shape[1])
        wm[f"target.L{l}.wqkv"] = torch.cat([W[:qd], k, v])
    for j in range(cfg.drafter.n_layers):
        wm[f"drafter.L{j}.wqkv"] = torch.zeros(cfg_m.drafter.qkv_dim, cfg.drafter.hidden)
    prompt = make_prompt("uniform", 10, d.vocab, 2)
    a = oracle.OracleSpec(cfg, w).session(32).prefill(prompt, want_logits=True)[2]
    b = oracle.OracleSpec(cfg_m, wm).session(32).prefill(prompt, want_logits=True)[2]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("case", ["fp32", "bf16", "moe", "block16", "qk_norm", "rope_scaled"])
def test_drafter_matches_dense_reference_through_rejections(case):
    """Drafter logits after several draft/verify/commit rounds equal a drafter
    whose context is rebuilt from scratch from the committed prefix: pins the
    fuse, the K/V injection and the rollback of rejected positions."""
    cfg = tiny(**CASES[case])
    w = make_weights(cfg, random_gains=True)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 9, cfg.target.vocab, 3)
    ss = spec.session(128)
    anchor, _, _ = ss.prefill(prompt)
    committed = list(prompt)
    ar = spec.generate_ar(prompt, 40)
    B = cfg.block_size
    rng = np.random.default_rng(11)
    for it in range(4):
        drafts, _, dl = ss.draft(anchor, want_logits=True)
        np.testing.assert_allclose(dl, dense_ref.drafter_block(cfg, w, committed, anchor), rtol=1e-9, atol=1e-9)
        # mix correct and wrong drafts so different accept lengths occur
        n_out = len(committed) - len(prompt) + 1
        script = list(ar[n_out:n_out + B - 1])
        cut = int(rng.integers(0, B))
        d = script[:cut] + [(x + 1) % cfg.target.vocab for x in script[cut:]]
        g, _, _ = ss.verify([anchor] + d)
        a = orc.accept(d, g, B)
        assert a == min(cut, B - 1)
        ss.commit(a)
        committed += [anchor] + d[:a]
        anchor = int(g[a])
        assert ss.len == len(committed)


@pytest.mark.parametrize("case", list(CASES) + ["block1", "block2"])
def test_spec_output_equals_target_only_greedy(case):
    kw = dict(CASES.get(case, {}))
    if case == "block1":
        kw = dict(block=1)
    if case == "block2":
        kw = dict(block=2)
    cfg = tiny(**kw)
    w = make_weights(cfg)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 16, cfg.target.vocab, 4)
    ar = spec.generate_ar(prompt, 48)
    out, acc = spec.generate_spec(prompt, 48)
    np.testing.assert_array_equal(out, ar)
    assert ((acc >= 0) & (acc <= cfg.block_size - 1)).all()


@pytest.mark.parametrize("case", ["fp32", "moe", "block16"])
def test_perfect_drafter_accepts_every_block(case):
    cfg = tiny(**CASES[case])
    w = make_weights(cfg)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 16, cfg.target.vocab, 5)
    B = cfg.block_size
    max_new = 1 + 3 * B
    ar = spec.generate_ar(prompt, max_new + B)
    out, acc = spec.generate_spec(prompt, max_new, forced=ar)
    np.testing.assert_array_equal(out, ar[:max_new])
    assert (acc == B - 1).all() and len(acc) == 3


def test_trained_like_drafter_partial_acceptance():
    """A script that is right for exactly k drafts gives a == k every iteration."""
    cfg = tiny(block=8)
    w = make_weights(cfg)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 16, cfg.target.vocab, 6)
    ar = spec.generate_ar(prompt, 80)
    B = cfg.block_size
    for k in (0, 3, 7):
        ss = spec.session(128)
        anchor, _, _ = ss.prefill(prompt)
        n_out = 1
        while n_out + B < 60:
            d = list(ar[n_out:n_out + B - 1])
            d = d[:k] + [(x + 1) % cfg.target.vocab for x in d[k:]]
            g, _, _ = ss.verify([anchor] + d)
            a = orc.accept(d, g, B)
            assert a == k
            ss.commit(a)
            n_out += a + 1
            anchor = int(g[a])
            assert anchor == ar[n_out - 1]


# ---------------------------------------------------------------- property: lossless for any shape
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=12, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(block=st.integers(1, 8), kv=st.sampled_from([(4, 1), (4, 2), (4, 4), (2, 2)]), moe=st.booleans(),
       taps=st.sampled_from([(0,), (1,), (0, 1), (1, 1, 0)]), t_layers=st.integers(1, 2),
       prompt_len=st.integers(1, 12), seed=st.integers(0, 10_000))
def test_spec_equals_target_only_for_random_shapes(block, kv, moe, taps, t_layers, prompt_len, seed):
    """Draft-and-verify output equals target-only greedy output bit for bit for any
    block size, GQA grouping, MoE routing, tap set and prompt; accept lengths stay
    in [0, block-1].  (Taps beyond the last layer are clamped to it.)"""
    nq, nkv = kv
    taps = tuple(min(t, t_layers - 1) for t in taps)
    cfg = tiny(block=block, nq=nq, nkv=nkv, moe=moe, taps=taps, t_layers=t_layers, vocab=256)
    spec = oracle.OracleSpec(cfg, make_weights(cfg, seed=seed))
    prompt = make_prompt("uniform", prompt_len, cfg.target.vocab, seed)
    ar = spec.generate_ar(prompt, 24)
    out, acc = spec.generate_spec(prompt, 24)
    np.testing.assert_array_equal(out, ar)
    assert ((acc >= 0) & (acc <= block - 1)).all()
