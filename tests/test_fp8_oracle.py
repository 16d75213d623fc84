"""Pins of the FP8 weight path, CPU only.

FP8 weights (E4M3 codes with one fp32 scale per output row, synthetic.fp8)
make a quantised model; the method run on it must reproduce that model's own
greedy decoding, so the oracle computes with the dequantised weights
scale * e4m3_value(code) in fp64.  Pinned by: the E4M3 codebook against
PyTorch's float8_e4m3fn conversion (all 256 codes); the encoder against
PyTorch's round-to-nearest-even cast, ties included; the quantiser's error
bound; the oracle's FP8 product against numpy on the dequantised matrix; the
oracle's FP8 target and drafter against the independent dense reference run on
the dequantised weights; and speculative output equal to target-only output.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from oracle import api as orc
from synthetic import get_config, make_prompt, make_weights
from synthetic.fast import make_weights_host
from synthetic.fp8 import dequantize_rows, e4m3_decode, e4m3_encode, quantize_rows

import dense_ref

ALL = torch.arange(256, dtype=torch.int32).to(torch.uint8)


def test_codebook_matches_torch_float8_e4m3fn():
    ref = ALL.view(torch.float8_e4m3fn).double()
    mine = e4m3_decode(ALL)
    orc_vals = torch.tensor([orc.e4m3_value(c) for c in range(256)], dtype=torch.float64)
    for v in (mine, orc_vals):
        assert torch.equal(torch.isnan(v), torch.isnan(ref))
        ok = ~torch.isnan(ref)
        assert torch.equal(v[ok], ref[ok])
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(0x01) == 2.0 ** -9 and orc.e4m3_value(0x08) == 2.0 ** -6


def test_encoder_rounds_like_torch_cast_ties_included():
    vals = e4m3_decode(ALL)
    ok = ~torch.isnan(vals)
    assert torch.equal(e4m3_encode(vals[ok].float()), ALL[ok])  # every code round-trips
    pos = vals[ok & (vals >= 0)].unique()
    mids = ((pos[1:] + pos[:-1]) / 2).float()                   # exact ties: to the even code
    g = torch.Generator().manual_seed(0)
    x = torch.cat([(torch.rand(200_000, generator=g, dtype=torch.float64) * 896 - 448).float(), mids, -mids,
                   torch.tensor([0.0, -0.0, 448.0, -448.0, 2.0 ** -10, 3 * 2.0 ** -10])])
    assert torch.equal(e4m3_encode(x), x.to(torch.float8_e4m3fn).view(torch.uint8))


def test_quantiser_error_bound():
    g = torch.Generator().manual_seed(1)
    w = (torch.randn(64, 512, generator=g) * 0.02).bfloat16()
    w[3] = 0                                                      # an all-zero row gets scale 1, codes 0
    codes, scale = quantize_rows(w)
    assert codes.dtype == torch.uint8 and scale.dtype == torch.float32
    wq = dequantize_rows(codes, scale)
    wd = w.double()
    assert torch.equal(wq[3], torch.zeros(512, dtype=torch.float64)) and scale[3] == 1
    amax = wd.abs().amax(-1)
    for r in range(64):
        if r == 3:
            continue
        # the largest element maps to +-448 (codes 0x7E / 0xFE)
        assert (codes[r] & 0x7F).max() == 0x7E
        # half a unit in the last place: 2^-4 relative above 2^-6 * scale, 2^-10 * scale below
        err = (wq[r] - wd[r]).abs()
        small = wd[r].abs() < 2.0 ** -6 * scale[r].double()
        assert (err[~small] <= 2.0 ** -4 * wd[r].abs()[~small] + 1e-30).all()
        assert (err[small] <= 2.0 ** -10 * scale[r].double() + 1e-30).all()
        assert abs(float(scale[r]) * 448 - float(amax[r])) <= 1e-6 * float(amax[r])


@pytest.mark.parametrize("N,K,R,row0", [(37, 200, 3, 0), (64, 1024, 5, 11)])
def test_oracle_fp8_product_is_the_dequantised_product(N, K, R, row0):
    g = torch.Generator().manual_seed(N + K)
    w = (torch.randn(N + row0, K, generator=g) * 0.02).bfloat16()
    codes, scale = quantize_rows(w)
    x = torch.randn(R, K, generator=g, dtype=torch.float64).numpy()
    got = orc.matmul_fp8(codes, scale, x, row0=row0, n_rows=N)
    want = x @ dequantize_rows(codes, scale).numpy()[row0:row0 + N].T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def _tiny_fp8(block=4, **kw):
    base = get_config("tiny")
    return base.with_(dtype="fp8", block_size=block, **kw)


def _dequantised(cfg, w):
    """The FP8 model's weights as fp64 dense tensors (names without .scale)."""
    out = {}
    for k, v in w.items():
        if k.endswith(".scale"):
            continue
        out[k] = dequantize_rows(v, w[k + ".scale"]) if v.dtype == torch.uint8 else v
    return out


def test_fp8_weights_host_and_torch_generators_agree():
    cfg = _tiny_fp8()
    a, b = make_weights(cfg), make_weights_host(cfg)
    assert a.keys() == b.keys()
    assert all(torch.equal(a[k], b[k]) for k in a)
    assert a["lm_head"].dtype == torch.uint8 and a["embed"].dtype == torch.bfloat16


@pytest.mark.parametrize("block", [4, 16])
def test_fp8_model_matches_dense_reference(block):
    cfg = _tiny_fp8(block)
    w = make_weights(cfg, random_gains=True)
    wd = _dequantised(cfg, w)
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


def test_fp8_spec_equals_target_only_and_differs_from_bf16():
    cfg = _tiny_fp8(block=4)
    w = make_weights(cfg)
    spec = oracle.OracleSpec(cfg, w)
    prompt = make_prompt("uniform", 16, cfg.target.vocab, 4)
    ar = spec.generate_ar(prompt, 40)
    out, acc = spec.generate_spec(prompt, 40)
    np.testing.assert_array_equal(out, ar)
    # the quantised model is a different model: its logits move by the quantisation error
    bf = get_config("tiny").with_(dtype="bf16", block_size=4)
    lb = oracle.OracleSpec(bf, make_weights(bf)).session(64).prefill(prompt, want_logits=True)[2]
    lq = spec.session(64).prefill(prompt, want_logits=True)[2]
    assert 1e-4 < np.abs(lb - lq).max() < 0.5
