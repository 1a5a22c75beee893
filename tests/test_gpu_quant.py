"""GPU parity of step 2 (context-derived scales and e4m3 quantisation): scales,
Q8, K8 and V8 (transposed layout, zero padding) bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import dev, host

pytestmark = pytest.mark.gpu


def _check(cuda_lib, orc, q_scaled, k, v, N):
    B, T, H, _ = q_scaled.shape
    q8, cache = cuda_lib.fp8_quantize_context(dev(q_scaled), dev(k), dev(v), N)
    torch.cuda.synchronize()
    assert cache.filled
    s_q, s_k, s_v = (orc.context_scales(x, N) for x in (q_scaled, k, v))
    sc = host(cache.scales)
    assert (sc[0] == s_q).all() and (sc[1] == s_k).all() and (sc[2] == s_v).all()
    assert (host(q8) == orc.quantize(q_scaled, s_q)).all()
    assert (host(cache.k8) == orc.quantize(k, s_k)).all()
    v8t = host(cache.v8t)
    want_v = orc.quantize(v, s_v)                        # [B,H,N,d]
    assert (v8t[..., :N] == want_v.transpose(0, 1, 3, 2)).all()
    assert (v8t[..., N:] == 0).all()


@pytest.mark.parametrize("B,N,M,H", [(1, 1024, 128, 4), (2, 1000, 77, 3), (1, 1, 0, 2), (1, 130, 1, 8)])
def test_quantize_bit_exact(cuda_lib, orc, B, N, M, H):
    inp = make_inputs(WORKLOADS["icl_n16k_m1k_h8"], n_ctx=N, n_query=M, heads=H, batch=B)
    qs = orc.qscale(inp["q"], N, inp["c_h"])
    _check(cuda_lib, orc, qs, inp["k"], inp["v"], N)


def test_quantize_with_outliers(cuda_lib, orc):
    inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=8192, n_query=256)
    qs = orc.qscale(inp["q"], 8192, inp["c_h"], inp["gate"])
    _check(cuda_lib, orc, qs, inp["k"], inp["v"], 8192)


def test_quotients_of_every_fp16_value(cuda_lib, orc):
    """Every finite fp16 value (up to each head's amax) divided by 256 different
    context scales, through the Q/K row and the transposed V quantisers: the
    e4m3 codes must equal those of an IEEE fp32 division in the oracle."""
    B, H = 4, 64
    vals = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)      # +0 .. 65504
    vals = np.concatenate([vals, -vals]).astype(np.float16)              # -0 too: its code is 0x80
    rows = (vals.size + 63) // 64
    flat = np.zeros(rows * 64, np.float16)
    flat[:vals.size] = vals
    rng = np.random.default_rng(42)
    # per-(b, h) amax: random fp16 magnitudes from subnormal to max
    amax = np.abs(rng.choice(vals[vals != 0], B * H)).astype(np.float16)
    x = np.empty((B, rows, H, 64), np.float16)
    base = flat.reshape(rows, 64).astype(np.float32)
    for i in range(B * H):
        b, h = divmod(i, H)
        a = np.float32(amax[i])
        x[b, :, h, :] = np.clip(base, -a, a).astype(np.float16)
    _check(cuda_lib, orc, x, x.copy(), x.copy(), rows)


def test_query_rows_above_the_context_amax_saturate(cuda_lib, orc):
    """Scales come from the context rows only, so query rows larger than every
    context value quantise to the saturated codes +-448 (0x7E / 0xFE); the codes
    match the oracle bit for bit and the layer's outputs for those rows stay
    within the gates."""
    from parity import AMB, gate
    N, M, H = 1000, 100, 3
    inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=N, n_query=M, heads=H)
    q = inp["q"].astype(np.float32)
    q[:, N:] *= 10.0                                           # queries up to 10x the context amax
    q = q.astype(np.float16)
    qs = orc.qscale(q, N, inp["c_h"])
    s_q = orc.context_scales(qs, N)
    want = orc.quantize(qs, s_q)
    sat = (want[:, :, N:] & 0x7F) == 0x7E
    assert sat.mean() > 0.2, "the construction saturates a large share of the query codes"
    q8, cache = cuda_lib.fp8_quantize_context(dev(qs), dev(inp["k"]), dev(inp["v"]), N)
    torch.cuda.synchronize()
    assert (host(q8) == want).all()
    out = cuda_lib.icl_attention(dev(q), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]))
    ref = orc.layer(q, inp["k"], inp["v"], N, inp["c_h"], **AMB)
    gate(host(out), ref["out"], ref["allow"], "saturated query rows")
