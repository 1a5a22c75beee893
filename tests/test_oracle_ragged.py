"""Pins of the oracle's ragged-batch composition (layer_ragged, attention_exact_ragged):
every estimator of a padded batch is the plain layer on its own unmasked rows, and
the padding rows can change nothing."""
import numpy as np
import pytest

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs


def small(B=3, N=300, M=20, H=2, gated=False):
    w = WORKLOADS["ragged_b16_n16k_m1k_h8"]
    inp = make_inputs(w, n_ctx=N, n_query=M, heads=H, batch=B)
    if gated:
        g = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=N, n_query=M, heads=H, batch=B)["gate"]
        inp["gate"] = g
    return inp


def test_full_lengths_equal_the_uniform_layer(orc):
    inp = small(gated=True)
    N = inp["N"]
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], [N] * inp["B"], inp["c_h"], inp["gate"])
    u = orc.layer(inp["q"], inp["k"], inp["v"], N, inp["c_h"], inp["gate"])
    assert np.array_equal(r["out16"].view(np.uint16), u["out16"].view(np.uint16))
    for key in ("s_q", "s_k", "s_v", "q8", "k8", "v8"):
        assert np.array_equal(r[key], u[key]), key


def test_padding_contents_cannot_change_anything(orc):
    inp = small()
    B, N, T = inp["B"], inp["N"], inp["q"].shape[1]
    lens = inp["ctx_len"]
    ref = orc.layer_ragged(inp["q"], inp["k"], inp["v"], lens, inp["c_h"])
    q, k, v = inp["q"].copy(), inp["k"].copy(), inp["v"].copy()
    for b, n in enumerate(lens):
        q[b, n:N] = np.float16(np.nan)
        k[b, n:] = np.float16(60000.0)
        v[b, n:] = np.float16(-np.inf)
    got = orc.layer_ragged(q, k, v, lens, inp["c_h"])
    assert np.array_equal(got["out16"].view(np.uint16), ref["out16"].view(np.uint16))
    for key in ("s_q", "s_k", "s_v", "q8", "k8", "v8"):
        assert np.array_equal(got[key], ref[key]), key
    for b, n in enumerate(lens):  # padding rows: zero outputs and zero codes
        assert not ref["out16"][b, n:N].any() and not ref["q8"][b][:, n:N].any()
        assert not ref["k8"][b][:, n:].any() and not ref["v8"][b][:, n:].any()


def test_each_estimator_is_the_layer_on_its_own_rows(orc):
    """Against the one-estimator layer on the rows written out by hand (context rows
    then query rows, as an unpadded problem of n_b + M rows)."""
    inp = small(B=2, N=257, M=9, H=3)
    lens = [129, 257]
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], lens, inp["c_h"])
    N = inp["N"]
    for b, n in enumerate(lens):
        q = np.concatenate([inp["q"][b:b + 1, :n], inp["q"][b:b + 1, N:]], axis=1)
        u = orc.layer(q, inp["k"][b:b + 1, :n].copy(), inp["v"][b:b + 1, :n].copy(), n, inp["c_h"])
        assert np.array_equal(r["out16"][b, :n], u["out16"][0, :n])
        assert np.array_equal(r["out16"][b, N:], u["out16"][0, n:])
        assert np.array_equal(r["s_q"][b], u["s_q"][0])


def test_batch_permutation(orc):
    inp = small(B=3)
    lens = np.array([300, 17, 151])
    perm = np.array([2, 0, 1])
    a = orc.layer_ragged(inp["q"], inp["k"], inp["v"], lens, inp["c_h"])
    b = orc.layer_ragged(inp["q"][perm], inp["k"][perm], inp["v"][perm], lens[perm], inp["c_h"])
    assert np.array_equal(a["out16"][perm].view(np.uint16), b["out16"].view(np.uint16))


def test_exact_ragged_matches_the_layer_without_quantisation(orc):
    """attention_exact_ragged on the scaled queries is close to the FP8 layer (it is
    the FP8 path's target) and zero on padding rows."""
    inp = small(B=2, N=200, M=10, H=2)
    lens = inp["ctx_len"]
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], lens, inp["c_h"])
    ex = orc.attention_exact_ragged(r["q_scaled"], inp["k"], inp["v"], lens)
    for b, n in enumerate(lens):
        assert not ex[b, n:200].any()
        rows = np.r_[0:n, 200:210]
        rel = np.sqrt(((r["out"][b, rows] - ex[b, rows]) ** 2).mean() / (ex[b, rows] ** 2).mean())
        assert rel < 0.2, rel


def test_lengths_must_fit(orc):
    inp = small(B=2, N=50, M=4)
    with pytest.raises(AssertionError):
        orc.layer_ragged(inp["q"], inp["k"], inp["v"], [0, 50], inp["c_h"])
    with pytest.raises(AssertionError):
        orc.layer_ragged(inp["q"], inp["k"], inp["v"], [51, 50], inp["c_h"])
