"""The attention kernel's FMA-pipe 2^x polynomial: the committed header matches
its Remez generator, and its float32 evaluation stays far inside the 1e-4
relative band in which the parity gate treats either e4m3 code as correct."""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "fp8_quant_logscale_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return [np.float32(float(v)) for v in re.findall(r"kExp2C\d = ([-0-9.e]+)f;", text)]


def test_header_matches_generator():
    gen = _gen()
    c, err = gen.remez()
    assert err < 3e-6
    assert _header_coeffs() == list(c.astype(np.float32))


def test_range_reduced_exp2_accuracy():
    """Emulate the kernel's steps in float32: clamp, round-to-integer trick, Horner, exponent add."""
    c = _header_coeffs()
    t = np.concatenate([np.linspace(-30, 0, 400001), -np.logspace(-8, 0, 2001), [0.0, 1e-7]]).astype(np.float32)
    r = (np.maximum(t, np.float32(-30)) + np.float32(12582912.0)).astype(np.float32)
    j = (r - np.float32(12582912.0)).astype(np.float32)
    f = (t - j).astype(np.float32)
    assert (np.abs(f) <= 0.5).all()
    q = np.full_like(f, c[4])
    for ci in (c[3], c[2], c[1], c[0]):
        q = (q.astype(np.float64) * f + ci).astype(np.float32)     # fma: one rounding
    bits = (q.view(np.uint32).astype(np.uint64) + (r.view(np.uint32).astype(np.uint64) << np.uint64(23))) % (1 << 32)
    p = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    rel = np.abs(p / np.exp2(t.astype(np.float64)) - 1)
    assert rel.max() < 1e-5
