"""Pins of the oracle's fp16 and e4m3 codecs (CPU only).

The e4m3 codec is checked against the format definition (hand-derived golden
values), exhaustive round trips, brute force at every rounding midpoint, and
torch's float8_e4m3fn cast (an independent library implementation of RNE);
the fp16 codec against numpy's float16 conversion.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _finite_codes(orc):
    c = np.arange(256, dtype=np.uint8)
    v = orc.e4m3_decode(c)
    return c[~np.isnan(v)], v[~np.isnan(v)]


def test_e4m3_golden_values(orc):
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e4m3_values.txt")) if ln.strip() and ln[0] != "#"]
    for code_hex, val in rows:
        code = int(code_hex, 16)
        got = orc.e4m3_decode(np.array([code], np.uint8))[0]
        assert got == float(val), (code_hex, got, val)
        assert np.signbit(got) == val.startswith("-")
        assert orc.e4m3_encode(np.array([float(val)]))[0] == code


def test_e4m3_all_codes_round_trip(orc):
    c = np.arange(256, dtype=np.uint8)
    v = orc.e4m3_decode(c)
    nan = np.isnan(v)
    assert set(c[nan].tolist()) == {0x7F, 0xFF}
    assert (orc.e4m3_encode(v[~nan]) == c[~nan]).all()
    assert (orc.e4m3_encode(np.array([np.nan]))[0]) == 0x7F
    assert np.nanmax(v) == 448.0 and np.nanmin(v) == -448.0


def test_e4m3_saturates(orc):
    big = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, np.inf])
    assert (orc.e4m3_encode(big) == 0x7E).all()
    assert (orc.e4m3_encode(-big) == 0xFE).all()


def test_e4m3_midpoints_ties_to_even(orc):
    c, v = _finite_codes(orc)
    pos = np.unique(v[v >= 0])
    mids = (pos[:-1] + pos[1:]) / 2
    enc = orc.e4m3_encode(mids)
    dec = orc.e4m3_decode(enc)
    lo, hi = pos[:-1], pos[1:]
    # each midpoint goes to the neighbour whose code (mantissa LSB) is even
    lo_code = orc.e4m3_encode(lo)
    want = np.where(lo_code % 2 == 0, lo, hi)
    assert (dec == want).all()
    # just off the midpoint: nearest wins
    assert (orc.e4m3_decode(orc.e4m3_encode(np.nextafter(mids, 0))) == lo).all()
    assert (orc.e4m3_decode(orc.e4m3_encode(np.nextafter(mids, np.inf))) == hi).all()
    # below half the smallest subnormal: zero, with the sign kept
    assert orc.e4m3_encode(np.array([2.0 ** -10]))[0] == 0x00
    assert orc.e4m3_encode(np.array([-1e-30]))[0] == 0x80


def test_e4m3_monotone(orc):
    y = np.linspace(-500, 500, 200001)
    d = orc.e4m3_decode(orc.e4m3_encode(y))
    assert (np.diff(d) >= 0).all()


def test_e4m3_matches_torch_cast(orc):
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.standard_normal(200000) * 50, rng.standard_normal(50000) * 1e-2,
                        rng.uniform(-448, 448, 50000)]).astype(np.float32)
    # torch does not saturate, so compare inside the finite range
    t = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = orc.e4m3_encode(y.astype(np.float64))
    inside = np.abs(y) < 448
    assert (ours[inside] == t[inside]).all()
    assert (orc.e4m3_decode(ours[~inside]) == np.sign(y[~inside]) * 448).all()


def test_f16_matches_numpy(orc):
    rng = np.random.default_rng(1)
    y = np.concatenate([rng.standard_normal(200000) * 1000, rng.standard_normal(100000) * 1e-6,
                        np.array([65504.0, 65519.99, 65520.0, 7e4, -7e4, 2.0 ** -25, 2.0 ** -24, 3 * 2.0 ** -26,
                                  0.0, -0.0])])
    want = y.astype(np.float16).view(np.uint16)
    got = orc.f16_encode(y)
    assert (got == want).all()
    h = np.arange(65536, dtype=np.uint16)
    dv = orc.f16_decode(h)
    ref = h.view(np.float16).astype(np.float64)
    same = (dv == ref) | (np.isnan(dv) & np.isnan(ref))
    assert same.all()


def test_f16_midpoints(orc):
    h = np.arange(0x0000, 0x7BFF, dtype=np.uint16)
    v = h.view(np.float16).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2
    want = mids.astype(np.float16).view(np.uint16)
    assert (orc.f16_encode(mids) == want).all()


@pytest.mark.parametrize("n", [1, 2, 3, 1000, 1024, 16384, 131072, 524288, 1 << 24])
def test_log_length_is_fp32_log(orc, n):
    lam = orc.log_length(n)
    exact = np.log(float(n))
    assert abs(lam - exact) <= np.spacing(np.float32(exact)) * 1.0
    assert orc.log_length(0) == 0.0  # clamped at n = 1
