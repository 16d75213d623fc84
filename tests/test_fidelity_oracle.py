"""Pins of the oracle's fidelity toggles (not on the pages), CPU only.

RoPE frequency rescaling in the Llama 3.1 form is pinned by what the rule
fixes: off, it leaves the rotation bit for bit unchanged; short wavelengths
keep their frequency, long ones are divided by the factor, the band between
lies strictly inside and meets both neighbours continuously; frequencies stay
non-increasing along the head; the rotation still depends on relative
position only and keeps norms.  QK-norm and both toggles end to end are pinned
against the dense reference and the lossless property in test_oracle_pins.
"""
import math
from dataclasses import replace

import numpy as np
import pytest

from oracle import api as orc
from synthetic import get_config

from test_oracle_pins import TINY_ROPE_SCALING


def _tiny_dims(scaling=TINY_ROPE_SCALING):
    return replace(get_config("tiny").target, rope_scaling=scaling)


def _base(d, i):
    return d.rope_theta ** (-2.0 * i / d.head_dim)


def test_rescaling_off_is_the_plain_rotation_bit_for_bit():
    rng = np.random.default_rng(0)
    for scaling in ((0.0, 0.0, 0.0, 0.0), (1.0, 1.0, 4.0, 256.0)):
        d = _tiny_dims(scaling)
        for pos in (0, 1, 17, 4095):
            v = rng.normal(size=d.head_dim)
            assert np.array_equal(orc.rope_dims(v, pos, d), orc.rope(v, pos, d.rope_theta))


def test_bands_of_the_tiny_rescaling():
    d = _tiny_dims()
    factor, low, high, orig = d.rope_scaling
    for i in range(d.head_dim // 2):
        f, base = orc.rope_inv_freq(d, i), _base(d, i)
        wavelen = 2 * math.pi / base
        if wavelen < orig / high:
            assert f == pytest.approx(base, rel=1e-15), i
        elif wavelen > orig / low:
            assert f == pytest.approx(base / factor, rel=1e-15), i
        else:
            assert base / factor < f < base, i
    kept = [i for i in range(32) if orc.rope_inv_freq(d, i) == pytest.approx(_base(d, i), rel=1e-15)]
    assert kept == list(range(9))  # the three bands all occur in the tiny model


def test_rescaling_is_continuous_at_both_band_edges():
    d0 = _tiny_dims()
    factor, low, high, _ = d0.rope_scaling
    i = 10
    wavelen = 2 * math.pi / _base(d0, i)
    for edge_orig, limit in ((wavelen * high, _base(d0, i)), (wavelen * low, _base(d0, i) / factor)):
        for eps in (-1e-9, 0.0, 1e-9):
            d = replace(d0, rope_scaling=(factor, low, high, edge_orig * (1 + eps)))
            assert orc.rope_inv_freq(d, i) == pytest.approx(limit, rel=1e-8)


@pytest.mark.parametrize("name", ["tiny", "llama31_8b"])
def test_frequencies_stay_non_increasing(name):
    d = get_config(name).target
    d = replace(d, rope_scaling=TINY_ROPE_SCALING if name == "tiny" else (8.0, 1.0, 4.0, 8192.0))
    f = [orc.rope_inv_freq(d, i) for i in range(d.head_dim // 2)]
    assert all(a >= b for a, b in zip(f, f[1:]))
    assert f[0] == 1.0


def test_published_llama31_setting_on_the_llama_shape():
    """theta 5e5, head_dim 128, factor 8, low 1, high 4, original 8192:
    wavelengths below 2048 keep their frequency, above 8192 are divided by 8."""
    d = replace(get_config("llama31_8b").target, rope_scaling=(8.0, 1.0, 4.0, 8192.0))
    assert d.rope_theta == 5e5 and d.head_dim == 128
    n_keep = n_div = n_mid = 0
    for i in range(64):
        base, f = _base(d, i), orc.rope_inv_freq(d, i)
        w = 2 * math.pi / base
        if w < 2048:
            n_keep += f == pytest.approx(base, rel=1e-15)
        elif w > 8192:
            n_div += f == pytest.approx(base / 8, rel=1e-15)
        else:
            n_mid += base / 8 < f < base
    assert n_keep + n_div + n_mid == 64 and min(n_keep, n_div, n_mid) > 0


def test_rescaled_rotation_depends_on_relative_position_only():
    d = _tiny_dims()
    rng = np.random.default_rng(1)
    q, k = rng.normal(size=d.head_dim), rng.normal(size=d.head_dim)
    for p, pk, shift in ((5, 2, 7), (40, 39, 100), (3, 3, 1000)):
        a = orc.rope_dims(q, p, d) @ orc.rope_dims(k, pk, d)
        b = orc.rope_dims(q, p + shift, d) @ orc.rope_dims(k, pk + shift, d)
        assert a == pytest.approx(b, rel=1e-10, abs=1e-10)
        assert np.linalg.norm(orc.rope_dims(q, p, d)) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    assert np.array_equal(orc.rope_dims(q, 0, d), q)
