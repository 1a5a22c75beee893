"""Pins of the ragged grouped-query prefill oracle (oracle.gqa_prefill) against the
C oracle's exact attention, closed forms and library casts."""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import PREFILL_WORKLOADS, bf16_bits, make_prefill_inputs


def test_bf16_codecs_against_torch(orc):
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 10.0 ** rng.integers(-3, 3, 4096),
                        np.array([0.0, -0.0, 1.0, -2.5, 65504.0, 1e-30, 3.3895314e38], np.float32)])
    bits = bf16_bits(x)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, want)
    dec = orc.bf16_decode(bits)
    assert np.array_equal(dec, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy())


def exact_inputs(rng, shape):
    """Values exactly representable in both fp16 and bf16: multiples of 1/16 in [-4, 4]."""
    x = (rng.integers(-64, 65, size=shape) / 16.0).astype(np.float32)
    return x, bf16_bits(x), x.astype(np.float16)


def test_non_causal_head_equals_the_c_exact_attention(orc):
    rng = np.random.default_rng(1)
    nq, nk, Hq, Hkv, d = 7, 33, 4, 2, 128
    _, qb, q16 = exact_inputs(rng, (nq, Hq, d))
    _, kb, k16 = exact_inputs(rng, (nk, Hkv, d))
    _, vb, v16 = exact_inputs(rng, (nk, Hkv, d))
    out = orc.gqa_prefill(qb, kb, vb, [0, nq], [0, nk], Hq, Hkv, causal=False)
    for h in range(Hq):
        g = h // 2
        ref = orc.attention_exact(q16[None, :, h:h + 1], k16[None, :, g:g + 1], v16[None, :, g:g + 1])
        assert np.allclose(out[:, h], ref[0, :, 0], rtol=0, atol=1e-12)


def test_causal_row_equals_attention_over_its_visible_keys(orc):
    rng = np.random.default_rng(2)
    nq, nk, Hq, Hkv, d = 5, 12, 2, 1, 128
    _, qb, q16 = exact_inputs(rng, (nq, Hq, d))
    _, kb, k16 = exact_inputs(rng, (nk, Hkv, d))
    _, vb, v16 = exact_inputs(rng, (nk, Hkv, d))
    out = orc.gqa_prefill(qb, kb, vb, [0, nq], [0, nk], Hq, Hkv, causal=True)
    for i in range(nq):
        vis = nk - nq + i + 1
        for h in range(Hq):
            ref = orc.attention_exact(q16[None, i:i + 1, h:h + 1], k16[None, :vis, 0:1], v16[None, :vis, 0:1])
            assert np.allclose(out[i, h], ref[0, 0, 0], rtol=0, atol=1e-12)


def test_closed_forms(orc):
    rng = np.random.default_rng(3)
    d, Hq, Hkv = 128, 8, 2
    # one query, one key: the output is that key's value row
    _, qb, _ = exact_inputs(rng, (1, Hq, d))
    _, kb, _ = exact_inputs(rng, (1, Hkv, d))
    x, vb, _ = exact_inputs(rng, (1, Hkv, d))
    out = orc.gqa_prefill(qb, kb, vb, [0, 1], [0, 1], Hq, Hkv)
    for h in range(Hq):
        assert np.array_equal(out[0, h], x[0, h // 4].astype(np.float64))
    # Q = 0, causal: each query averages the values it can see
    nq, nk = 6, 20
    zq = bf16_bits(np.zeros((nq, Hq, d), np.float32))
    _, kb, _ = exact_inputs(rng, (nk, Hkv, d))
    x, vb, _ = exact_inputs(rng, (nk, Hkv, d))
    out = orc.gqa_prefill(zq, kb, vb, [0, nq], [0, nk], Hq, Hkv)
    for i in range(nq):
        vis = nk - nq + i + 1
        for h in range(Hq):
            assert np.allclose(out[i, h], x[:vis, h // 4].astype(np.float64).mean(axis=0), atol=1e-12)


def test_grouped_heads_and_sequence_independence(orc):
    inp = make_prefill_inputs(PREFILL_WORKLOADS["gqa4_prefill_b2"], q_lens=(5, 9), kv_lens=(40, 70))
    q = inp["q"].copy()
    q[:, 1] = q[:, 0]       # heads 0 and 1 share key/value head 0 and now their queries
    args = (inp["qo_indptr"], inp["kv_indptr"], 16, 4)
    out = orc.gqa_prefill(q, inp["k"], inp["v"], *args)
    assert np.array_equal(out[:, 0], out[:, 1])
    k = inp["k"].copy()
    k[40:] = bf16_bits(np.full(k[40:].shape, 3.0, np.float32))   # sequence 1's keys only
    out2 = orc.gqa_prefill(q, k, inp["v"], *args)
    assert np.array_equal(out2[:5], out[:5]) and not np.array_equal(out2[5:], out[5:])


def test_causal_needs_enough_keys(orc):
    inp = make_prefill_inputs(PREFILL_WORKLOADS["gqa4_prefill_b2"], q_lens=(5,), kv_lens=(4,))
    with pytest.raises(AssertionError):
        orc.gqa_prefill(inp["q"], inp["k"], inp["v"], inp["qo_indptr"], inp["kv_indptr"], 16, 4)
