"""Pins of the MXFP4 weight path, CPU only.

MXFP4 weights (packed E2M1 codes sharing one power-of-two exponent per 32
values along K, plus one fp32 scale per row; synthetic.fp4) make a quantised
model; the method run on it must reproduce that model's own greedy decoding,
so the oracle computes with the dequantised weights in fp64.  Pinned by: the
E2M1 codebook against the published table (tests/golden/e2m1_values.txt); the
UE8M0 block exponents against PyTorch's float8_e8m0fnu conversion; the encoder
against a brute-force nearest search with the ties-to-even rule; the
quantiser's block exponent rule and error bound; the oracle's MXFP4 product
against numpy on the dequantised matrix; the oracle's MXFP4 target and drafter
against the independent dense reference run on the dequantised weights; and
speculative output equal to target-only output.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import api as orc
from synthetic import get_config, make_prompt, make_weights
from synthetic.fast import make_weights_host
from synthetic.fp4 import block_exponents, dequantize_mx, e2m1_decode, e2m1_encode, quantize_mx, unpack_codes

import dense_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_values.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        code, val = (x.strip() for x in line.split("|"))
        out[int(code, 2)] = float(val)
    return out


def test_codebook_matches_published_table():
    g = _golden()
    assert sorted(g) == list(range(16))
    mine = e2m1_decode(torch.arange(16))
    for c, v in g.items():
        assert mine[c].item() == v and orc.e2m1_value(c) == v
        assert np.signbit(orc.e2m1_value(c)) == np.signbit(v)  # -0.0 keeps its sign


def test_block_exponent_bytes_decode_like_torch_e8m0():
    b = torch.arange(255, dtype=torch.int32).to(torch.uint8)  # 255 is E8M0's NaN, never produced
    ref = b.view(torch.float8_e8m0fnu).double()
    codes = torch.full((1, 64), 0x22, dtype=torch.uint8)        # every element 1.0
    for e in range(0, 255, 17):
        bs = torch.full((1, 1, 4), e, dtype=torch.uint8)
        w = dequantize_mx(codes, bs, torch.ones(1))
        assert torch.equal(w, torch.full((1, 128), ref[e].item(), dtype=torch.float64))


def _nearest_even(y: float) -> int:
    """Brute force: the E2M1 code nearest to y (saturating), ties to the even code."""
    grid = [e2m1_decode(torch.tensor(c)).item() for c in range(8)]
    a = min(abs(y), 6.0)
    d = [abs(a - v) for v in grid]
    best = min(d)
    cands = [c for c in range(8) if d[c] == best]
    c = cands[0] if len(cands) == 1 else [x for x in cands if x % 2 == 0][0]
    return c | (8 if np.signbit(y) else 0)


def test_encoder_is_nearest_with_ties_to_even_and_saturates():
    vals = e2m1_decode(torch.arange(16)).float()
    assert torch.equal(e2m1_encode(vals), torch.arange(16).to(torch.uint8))   # every code round-trips
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.rand(3000, generator=g) * 16 - 8, mids, -mids, torch.tensor([7.9, -100.0, 6.0001, 1e-30])])
    got = e2m1_encode(x.float())
    want = torch.tensor([_nearest_even(v) for v in x.tolist()], dtype=torch.uint8)
    assert torch.equal(got, want)


def test_quantiser_block_exponents_and_error_bound():
    g = torch.Generator().manual_seed(1)
    w = (torch.randn(24, 512, generator=g) * 0.02).bfloat16()
    w[3] = 0                                   # all-zero rows: exponent byte 0, codes 0
    w[5, 32:64] = 0                            # one all-zero block
    codes, bscale, scale = quantize_mx(w)
    assert codes.shape == (24, 256) and bscale.shape == (4, 24, 4) and torch.equal(scale, torch.ones(24))
    wd = w.double()
    wq = dequantize_mx(codes, bscale, scale)
    assert torch.equal(wq[3], torch.zeros(512, dtype=torch.float64))
    assert (bscale[:, 3, :] == 0).all() and bscale[0, 5, 1] == 0
    E = block_exponents(w)
    for r in range(24):
        for b in range(16):
            blk = wd[r, 32 * b:32 * b + 32]
            amax = blk.abs().max().item()
            e = int(bscale[b // 4, r, b % 4]) - 127
            assert e == E[r, b]
            if amax == 0:
                continue
            assert 2.0 ** (e + 2) <= amax < 2.0 ** (e + 3)              # the largest element lands in [4, 8)
            err = (wq[r, 32 * b:32 * b + 32] - blk).abs()
            assert (err < 2.0 ** (e + 1)).all()                              # saturation at 6: below 8 - 6
            # below the saturation point the error is at most half a grid step: 1 * 2^e
            unsat = blk.abs() <= 6 * 2.0 ** e
            assert (err[unsat] <= 2.0 ** e).all()
    # the codes' nibbles unpack in element order
    assert torch.equal(unpack_codes(codes)[:, 0::2], codes & 15)


@pytest.mark.parametrize("N,K,R,row0", [(37, 256, 3, 0), (64, 1024, 5, 11)])
def test_oracle_mxfp4_product_is_the_dequantised_product(N, K, R, row0):
    g = torch.Generator().manual_seed(N + K)
    w = (torch.randn(N + row0, K, generator=g) * 0.02).bfloat16()
    codes, bscale, scale = quantize_mx(w)
    scale = torch.rand(N + row0, generator=g) + 0.5          # any row scale, not only 1
    x = torch.randn(R, K, generator=g, dtype=torch.float64).numpy()
    got = orc.matmul_mxfp4(codes, bscale, scale, x, row0=row0, n_rows=N)
    want = x @ dequantize_mx(codes, bscale, scale).numpy()[row0:row0 + N].T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def _tiny_fp4(block=4, **kw):
    return get_config("tiny").with_(dtype="fp4", block_size=block, **kw)


def _dequantised(w):
    out = {}
    for k, v in w.items():
        if k.endswith(".scale") or k.endswith(".bscale"):
            continue
        out[k] = dequantize_mx(v, w[k + ".bscale"], w[k + ".scale"]) if v.dtype == torch.uint8 else v
    return out


def test_fp4_weights_host_and_torch_generators_agree():
    cfg = _tiny_fp4()
    a, b = make_weights(cfg), make_weights_host(cfg)
    assert a.keys() == b.keys()
    assert all(torch.equal(a[k], b[k]) for k in a)
    assert a["lm_head"].dtype == torch.uint8 and a["lm_head"].shape == (cfg.target.vocab, cfg.target.hidden // 2)
    assert a["embed"].dtype == torch.bfloat16


@pytest.mark.parametrize("block", [4, 16])
def test_fp4_model_matches_dense_reference(block):
    cfg = _tiny_fp4(block)
    w = make_weights(cfg, random_gains=True)
    wd = _dequantised(w)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 12, cfg.target.vocab, 1)
    ss = spec.session(96)
    anchor, _, lg0 = ss.prefill(prompt, want_logits=True)
    ref, _ = dense_ref.target_forward(cfg, wd, list(prompt))
    np.testing.assert_allclose(lg0, ref[-1], rtol=1e-9, atol=1e-9)
    _, _, dl = ss.draft(anchor, want_logits=True)
    np.testing.assert_allclose(dl, dense_ref.drafter_block(cfg, wd, list(prompt), anchor), rtol=1e-9, atol=1e-9)
    blk = [anchor] + list(range(1, block))
    _, _, lg = ss.verify(blk, want_logits=True)
    ref, _ = dense_ref.target_forward(cfg, wd, list(prompt) + blk)
    np.testing.assert_allclose(lg, ref[len(prompt):], rtol=1e-9, atol=1e-9)


def test_fp4_spec_equals_target_only_and_differs_from_fp8():
    cfg = _tiny_fp4(block=4)
    w = make_weights(cfg)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 16, cfg.target.vocab, 4)
    ar = spec.generate_ar(prompt, 40)
    out, acc = spec.generate_spec(prompt, 40)
    np.testing.assert_array_equal(out, ar)
    # the 4-bit model is a different model from the 8-bit one: its logits move
    f8 = get_config("tiny").with_(dtype="fp8", block_size=4)
    l8 = oracle.OracleSpec(f8, make_weights(f8)).session(64).prefill(prompt, want_logits=True)[2]
    l4 = spec.session(64).prefill(prompt, want_logits=True)[2]
    assert 1e-4 < np.abs(l8 - l4).max() < 2.0
