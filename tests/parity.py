"""Teacher-forced parity protocol between the CUDA library and the fp64 oracle.

The GPU drives the sequence; the oracle replays the same committed tokens and
the same GPU drafts, and recomputes its own logits and argmaxes.  Checks:
  1. every drafter / target logit row within `tol` of the oracle's;
  2. every GPU draft and target argmax equals the oracle's, unless the
     oracle's top-1/top-2 margin there is below `tie` (counted);
  3. the accept length, committed tokens and new length equal the greedy rule
     applied to the GPU's own drafts and argmaxes -- always bit-exact;
  4. they also equal the rule applied to the oracle's argmaxes unless a
     counted near-tie sits at an index <= a.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

import numpy as np
import torch

import block_diffusion_speculative_layers_b200 as dfl
import oracle
from oracle import api as orc
from synthetic import make_weights
from synthetic.fast import make_weights_host


@dataclass
class Report:
    max_dlogit: float = 0.0
    near_ties: int = 0
    checked_tokens: int = 0
    accepts: List[int] = field(default_factory=list)
    mismatches_outside_ties: int = 0
    sessions: list = field(default_factory=list)


def accept_rule(drafts, g) -> int:
    a = 0
    while a < len(drafts) and drafts[a] == g[a]:
        a += 1
    return a


def build_pair(cfg, max_batch=1, max_len=256, random_gains=True, prefill_chunk=0, seed=None):
    w_cpu = make_weights_host(cfg, random_gains=random_gains, seed=seed)
    gpu = dfl.DFlash(cfg, max_batch=max_batch, max_len=max_len, prefill_chunk=prefill_chunk, keep_logits=True)
    w_gpu = make_weights(cfg, device="cuda", random_gains=random_gains, seed=seed)
    gpu.load_weights(w_gpu)
    spec = oracle.OracleSpec(cfg, w_cpu)
    return gpu, spec, w_cpu


def _cmp_tokens(gpu_tok, orc_tok, margins, tie, rep: Report):
    ties_at = []
    for i, (a, b) in enumerate(zip(gpu_tok, orc_tok)):
        rep.checked_tokens += 1
        if a != b:
            if margins[i] < tie:
                rep.near_ties += 1
                ties_at.append(i)
            else:
                rep.mismatches_outside_ties += 1
        elif margins[i] < tie:
            ties_at.append(i)
    return ties_at


def replay(gpu, spec, cfg, prompts, n_iters, tol, tie, seqs=None) -> Report:
    """Prefill each prompt (slot = index), then n_iters draft/verify iterations over all."""
    rep = Report()
    B = cfg.block_size
    n = len(prompts)
    seqs = list(range(n)) if seqs is None else list(seqs)
    sess, anchors = [], []
    for i, p in enumerate(prompts):
        first = gpu.prefill(seqs[i], p)
        lg = gpu.debug_logits(2, 1)[0]
        ss = spec.session(len(p) + (n_iters + 2) * B + 8)
        tok_o, mg, lg_o = ss.prefill(p, want_logits=True)
        rep.max_dlogit = max(rep.max_dlogit, float(np.abs(lg - lg_o).max()))
        _cmp_tokens([first], [tok_o], [mg], tie, rep)
        assert int(np.argmax(lg)) == first
        sess.append(ss)
        anchors.append(first)
    for it in range(n_iters):
        d_gpu = gpu.draft_block(seqs)                       # [n, B-1]
        dl = gpu.debug_logits(0, n * B).reshape(n, B, -1) if B > 1 else None
        for i in range(n):
            if B > 1:
                d_o, mg_d, dl_o = sess[i].draft(anchors[i], want_logits=True)
                rep.max_dlogit = max(rep.max_dlogit, float(np.abs(dl[i, 1:] - dl_o).max()))
                assert (np.argmax(dl[i, 1:], axis=-1) == d_gpu[i]).all()
                _cmp_tokens(d_gpu[i], d_o, mg_d, tie, rep)
        acc, com, nl = gpu.verify_commit(seqs)
        vl = gpu.debug_logits(1, n * B).reshape(n, B, -1)
        for i in range(n):
            blk = [anchors[i]] + list(d_gpu[i])
            g_o, mg_v, vl_o = sess[i].verify(blk, want_logits=True)
            rep.max_dlogit = max(rep.max_dlogit, float(np.abs(vl[i] - vl_o).max()))
            g_gpu = np.argmax(vl[i], axis=-1)
            ties = _cmp_tokens(g_gpu, g_o, mg_v, tie, rep)
            a = int(acc[i])
            # (3) integer rule on the GPU's own values: always exact
            assert a == accept_rule(list(d_gpu[i]), list(g_gpu)), (it, i)
            want = list(d_gpu[i][:a]) + [int(g_gpu[a])]
            assert list(com[i][:a + 1]) == want
            assert int(nl[i]) == sess[i].len + a + 1
            # (4) against the oracle's argmaxes unless a near-tie at index <= a
            a_o = accept_rule(list(d_gpu[i]), list(g_o))
            if a_o != a:
                assert any(t <= min(a, a_o) for t in ties), (it, i, a, a_o, ties)
            sess[i].commit(a)
            anchors[i] = int(g_gpu[a])
            rep.accepts.append(a)
    rep.sessions = sess
    return rep


def check_lossless_generate(gpu, spec, cfg, prompt, max_new, tie):
    """GPU draft-and-verify output == oracle target-only greedy output up to the
    first divergence, which must sit at a near-tie of the oracle."""
    out, st = gpu.generate([prompt], max_new)
    ar, margins = spec.generate_ar(prompt, max_new, with_margins=True)
    out = out[0]
    div = np.nonzero(out != ar)[0]
    if len(div):
        k = int(div[0])
        assert margins[k] < tie, (k, out[:k + 2], ar[:k + 2], margins[k])
        return k, st
    return None, st


def replay_forced(gpu, spec, cfg, prompt, cuts, tol, tie, seq=0, check_kv=True, kv_tol=1e-2):
    """Greedy acceptance at chosen lengths: the caller's drafts are the oracle's
    own target-only continuation, made wrong at draft k+1 (none wrong for
    k = B-1), so the verify must accept exactly k drafts and commit k+1 tokens
    -- unless a counted near-tie of the oracle sits at an index <= k.  Each
    iteration checks the drafter and verify logits against the oracle replaying
    the same block, the accept length / committed tokens / new length bit for
    bit against the rule on the GPU's own argmaxes, the committed tokens against
    the oracle's continuation, and the target K/V of the committed positions
    and the drafter context K/V injected for them against the oracle's."""
    rep = Report()
    B, V = cfg.block_size, cfg.target.vocab
    n_ar = 1 + sum(k + 1 for k in cuts) + B
    ar, ar_mg = spec.generate_ar(prompt, n_ar, with_margins=True)
    ss = spec.session(len(prompt) + n_ar + 2 * B)
    first = gpu.prefill(seq, prompt)
    tok_o, mg, lg_o = ss.prefill(prompt, want_logits=True)
    lg = gpu.debug_logits(2, 1)[0]
    rep.max_dlogit = max(rep.max_dlogit, float(np.abs(lg - lg_o).max()))
    assert first == tok_o or mg < tie
    assert first == ar[0] or ar_mg[0] < tie
    j = 0  # index of the anchor in the continuation
    anchor = first
    for k in cuts:
        assert 0 <= k <= B - 1
        d_gpu = gpu.draft_block([seq])[0]
        if B > 1:
            d_o, mg_d, dl_o = ss.draft(anchor, want_logits=True)
            dl = gpu.debug_logits(0, B)[1:]
            rep.max_dlogit = max(rep.max_dlogit, float(np.abs(dl - dl_o).max()))
            _cmp_tokens(d_gpu, d_o, mg_d, tie, rep)
        drafts = [int(t) for t in ar[j + 1:j + B]]
        if k < B - 1:
            drafts[k] = (drafts[k] + 1) % V
        p0 = ss.len
        acc, com, nl = gpu.verify_commit([seq], drafts=np.array(drafts, np.int32).reshape(1, -1))
        vl = gpu.debug_logits(1, B)
        g_o, mg_v, vl_o = ss.verify([anchor] + drafts, want_logits=True)
        rep.max_dlogit = max(rep.max_dlogit, float(np.abs(vl - vl_o).max()))
        g_gpu = np.argmax(vl, axis=-1)
        ties = _cmp_tokens(g_gpu, g_o, mg_v, tie, rep)
        a = int(acc[0])
        assert a == accept_rule(drafts, list(g_gpu)), (k, a)
        assert list(com[0][:a + 1]) == drafts[:a] + [int(g_gpu[a])]
        assert int(nl[0]) == p0 + a + 1
        if a != k:  # only an oracle near-tie at an index <= k may shorten the block
            assert any(t <= k for t in ties), (k, a, ties)
        else:
            want = [int(t) for t in ar[j + 1:j + k + 2]]
            got = [int(t) for t in com[0][:a + 1]]
            if got != want:  # continuation and block verify may round a near-tie differently
                bad = [i for i in range(a + 1) if got[i] != want[i]]
                assert mg_v[bad[0]] < tie, (k, got, want)
        ss.commit(a)
        rep.accepts.append(a)
        if check_kv:
            for layer in sorted({0, cfg.target.n_layers - 1}):
                kg, vg = gpu.debug_kv(0, layer, seq, p0, a + 1)
                for t in range(a + 1):
                    ko, vo = ss.target_kv(layer, p0 + t)
                    assert np.abs(kg[t] - ko).max() <= kv_tol and np.abs(vg[t] - vo).max() <= kv_tol, (k, layer, t)
        anchor = int(g_gpu[a])
        if a != k or [int(t) for t in com[0][:a + 1]] != [int(t) for t in ar[j + 1:j + k + 2]]:
            break  # the GPU left the oracle's continuation at a near-tie: stop forcing
        j += a + 1
    if check_kv and B > 1 and rep.accepts:
        # the context rows of the last commit are injected by the next draft
        a = rep.accepts[-1]
        p0 = ss.len - (a + 1)
        gpu.draft_block([seq])
        ss.draft(anchor)
        for layer in range(cfg.drafter.n_layers):
            kg, vg = gpu.debug_kv(1, layer, seq, p0, a + 1)
            for t in range(a + 1):
                ko, vo = ss.ctx_kv(layer, p0 + t)
                assert np.abs(kg[t] - ko).max() <= kv_tol and np.abs(vg[t] - vo).max() <= kv_tol, (layer, t)
    rep.sessions = [ss]
    return rep
