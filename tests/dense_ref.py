"""An independent dense-matrix restatement of the model, used to pin the oracle.

The oracle (oracle/dflash_oracle.c) works row by row with a KV cache.  This
module computes the same definitions in whole-sequence matrix form: the target
over a full token prefix with an explicit causal mask matrix, and a drafter
block whose context keys are recomputed from scratch from that prefix.  It
shares no code with the oracle (numpy only) and is only used in tests on tiny
models.
"""
from __future__ import annotations

import numpy as np
import torch


def _np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, np.float64)


def rms(x, g, eps):
    return x / np.sqrt((x * x).mean(-1, keepdims=True) + eps) * g


def inv_freq(d):
    """RoPE inverse frequencies of model shape d; with d.rope_scaling's factor
    above 1, bands by wavelength: short ones kept, long ones divided by the
    factor, the ones between mixed linearly in original_max / wavelength."""
    hd = d.head_dim
    f = d.rope_theta ** (-np.arange(hd // 2, dtype=np.float64) * 2.0 / hd)
    factor, low, high, orig = d.rope_scaling
    if factor <= 1.0:
        return f
    ratio = orig / (2.0 * np.pi / f)                  # how many wavelengths fit the original window
    w = np.clip((ratio - low) / (high - low), 0.0, 1.0)  # 1: keep f, 0: f / factor
    return w * f + (1.0 - w) * f / factor


def rope(x, pos, d):
    """x [..., T, hd]; rotate-half pairing with the frequencies of model shape d."""
    hd = x.shape[-1]
    half = hd // 2
    freq = inv_freq(d)
    ang = np.asarray(pos, np.float64)[:, None] * freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def softmax(s, axis=-1):
    m = s.max(axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=axis, keepdims=True)


def silu(x):
    return x / (1.0 + np.exp(-x))


def _moe(d, W, p, m):
    E, K = d.n_experts, d.top_k
    Wr = _np(W[p + "w_router"])
    Wgu = _np(W[p + "we_gate_up"])
    Wd = _np(W[p + "we_down"])
    probs = softmax(m @ Wr.T, -1)                        # [T, E]
    out = np.zeros_like(m)
    Fe = d.expert_ffn
    for t in range(m.shape[0]):
        order = np.lexsort((np.arange(E), -probs[t]))    # by prob desc, then index asc
        sel = order[:K]
        w = probs[t, sel] / probs[t, sel].sum()
        for wi, e in zip(w, sel):
            gu = Wgu[e] @ m[t]
            out[t] += wi * (Wd[e] @ (silu(gu[:Fe]) * gu[Fe:]))
    return out


def _layer(d, W, p, x, pos, keys_extra=None, mask=None):
    """One pre-norm decoder layer over rows x [T, H] at positions pos.

    keys_extra: optional (K_ctx [nkv, C, hd], V_ctx) prepended to the rows' own keys.
    mask: boolean [T, C + T] of allowed (query, key) pairs.
    """
    T = x.shape[0]
    nq, nkv, hd = d.n_q_heads, d.n_kv_heads, d.head_dim
    qd, kd = nq * hd, nkv * hd
    n = rms(x, _np(W[p + "attn_norm"]), d.rms_eps)
    qkv = n @ _np(W[p + "wqkv"]).T
    q = qkv[:, :qd].reshape(T, nq, hd).transpose(1, 0, 2)
    k = qkv[:, qd:qd + kd].reshape(T, nkv, hd).transpose(1, 0, 2)
    v = qkv[:, qd + kd:].reshape(T, nkv, hd).transpose(1, 0, 2)
    if d.qk_norm:                           # per-head RMSNorm of q and k before RoPE
        q = rms(q, _np(W[p + "q_norm"]), d.rms_eps)
        k = rms(k, _np(W[p + "k_norm"]), d.rms_eps)
    q = rope(q, pos, d)
    k = rope(k, pos, d)
    if keys_extra is not None:
        k = np.concatenate([keys_extra[0], k], axis=1)
        v = np.concatenate([keys_extra[1], v], axis=1)
    grp = nq // nkv
    k = np.repeat(k, grp, axis=0)          # q head h uses kv head h // grp
    v = np.repeat(v, grp, axis=0)
    s = q @ k.transpose(0, 2, 1) / np.sqrt(hd)
    s = np.where(mask[None], s, -np.inf)
    o = (softmax(s, -1) @ v).transpose(1, 0, 2).reshape(T, qd)
    x = x + o @ _np(W[p + "wo"]).T
    m = rms(x, _np(W[p + "ffn_norm"]), d.rms_eps)
    if d.n_experts > 0:
        x = x + _moe(d, W, p, m)
    else:
        gu = m @ _np(W[p + "w_gate_up"]).T
        F = d.ffn
        x = x + (silu(gu[:, :F]) * gu[:, F:]) @ _np(W[p + "w_down"]).T
    return x


def target_forward(cfg, W, tokens):
    """Causal target over the whole prefix.  Returns (logits [T, V], taps {layer: [T, H]})."""
    d = cfg.target
    tokens = np.asarray(tokens)
    T = len(tokens)
    x = _np(W["embed"])[tokens]
    pos = np.arange(T)
    mask = np.tril(np.ones((T, T), bool))
    taps = {}
    for l in range(d.n_layers):
        x = _layer(d, W, f"target.L{l}.", x, pos, mask=mask)
        taps[l] = x.copy()
    logits = rms(x, _np(W["target.final_norm"]), d.rms_eps) @ _np(W["lm_head"]).T
    return logits, taps


def context(cfg, W, taps, n_pos):
    """Fused context vectors c_t for t < n_pos from target taps."""
    z = np.concatenate([taps[l][:n_pos] for l in cfg.tap_layers], axis=-1)
    return rms(z @ _np(W["fuse.w_fc"]).T, _np(W["fuse.norm"]), cfg.drafter.rms_eps)


def drafter_block(cfg, W, committed, anchor):
    """Drafter logits for block rows 1..B-1 given committed tokens [0, p) and the anchor at p."""
    d = cfg.drafter
    B = cfg.block_size
    committed = np.asarray(committed)
    p = len(committed)
    _, taps = target_forward(cfg, W, committed)
    c = context(cfg, W, taps, p)                      # [p, H]
    nkv, hd = d.n_kv_heads, d.head_dim
    qd, kd = d.n_q_heads * hd, nkv * hd
    toks = np.array([anchor] + [cfg.mask_id] * (B - 1))
    x = _np(W["embed"])[toks]
    pos = np.arange(p, p + B)
    mask = np.ones((B, p + B), bool)                  # block-bidirectional
    for j in range(d.n_layers):
        wqkv = _np(W[f"drafter.L{j}.wqkv"])
        kc = (c @ wqkv[qd:qd + kd].T).reshape(p, nkv, hd).transpose(1, 0, 2)
        vc = (c @ wqkv[qd + kd:].T).reshape(p, nkv, hd).transpose(1, 0, 2)
        if d.qk_norm:
            kc = rms(kc, _np(W[f"drafter.L{j}.k_norm"]), d.rms_eps)
        kc = rope(kc, np.arange(p), d)
        x = _layer(d, W, f"drafter.L{j}.", x, pos, keys_extra=(kc, vc), mask=mask)
    logits = rms(x, _np(W["drafter.final_norm"]), d.rms_eps) @ _np(W["lm_head"]).T
    return logits[1:]
