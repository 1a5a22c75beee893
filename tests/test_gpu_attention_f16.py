"""GPU parity of the normal-precision (fp16 tensor-core) ICL attention against
the oracle's double-precision attention of the same query-scaled inputs, and
the precision rule's dispatch.

The kernel's arithmetic fixes the tolerance (f16_bound): fp16 q', k, v;
fp32 logits from the tensor core (64 exact products summed in fp32); 2^x from
the MUFU or the degree-4 polynomial (relative error < 3e-6); probabilities
rounded to fp16 for the P.V product (relative 2^-11, absolute 2^-25 below
2^-14) while the row sum adds them unrounded; fp32 accumulation of O and l;
one fp16 rounding of the output.  Per (row, head), with S the largest
sum_e |q'_e k_e| over the keys and c2 = log2(e)/8:
    eta   = ln2 * c2 * S * 2^-17 + 3e-6        (logit and 2^x error of each p)
    bound = vmax * (2^-11 + 2 eta + N 2^-25 + (N/16 + N/8) 2^-23) + 1 fp16 ulp
where vmax is the largest |v| of the head; every element must lie within it,
and the mean error within 1/16 of the mean bound (a correct kernel's is
about 1/100: the per-key errors are independent roundings).
"""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import dev, fp16_ulp, host

pytestmark = pytest.mark.gpu
C2 = 1.4426950408889634 / 8.0


def f16_bound(qs, k, v, rows, exact):
    """Elementwise error bound [B, n, H, 64] of the fp16 kernel against exact attention."""
    B, _, H, d = qs.shape
    N = k.shape[1]
    bound = np.empty(exact.shape, np.float64)
    for b in range(B):
        for h in range(H):
            qa = np.abs(qs[b, rows, h].astype(np.float64))
            ka = np.abs(k[b, :, h].astype(np.float64))
            s_max = (qa @ ka.T).max(axis=1)                       # [n]
            eta = np.log(2.0) * C2 * s_max * 2.0 ** -17 + 3e-6
            vmax = float(np.abs(v[b, :, h].astype(np.float64)).max())
            rel = 2.0 ** -11 + 2 * eta + N * 2.0 ** -25 + (N / 16 + N / 8) * 2.0 ** -23
            bound[b, :, h, :] = (vmax * rel)[:, None]
    return bound + fp16_ulp(exact)


def check_f16(got, exact, bound, what):
    g = got.astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    d = np.abs(g - exact)
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()), max_ratio=float((d / bound).max()),
                 mean_bound=float(bound.mean()), n=int(d.size))
    print(f"\n{what}: {stats}")
    assert (d <= bound).all(), f"{what}: |d| above the bound ({stats})"
    assert d.mean() <= bound.mean() / 16, f"{what}: mean |d| too large ({stats})"
    return stats


def run_f16(cuda_lib, inp, gated, scaled=True):
    B, N, M, H = inp["B"], inp["N"], inp["M"], inp["H"]
    g = inp["gate"] if gated else None
    ws = cuda_lib.new_workspace(cuda_lib.workspace_size(cuda_lib.OP_ICL_ATTENTION_F16, B, N, M, H), "cuda")
    out = cuda_lib.icl_attention_f16(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N,
                                     dev(inp["c_h"]) if scaled else None, dev(g), ws=ws)
    st, flags = cuda_lib.sync_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    return host(out)


def layer_case(cuda_lib, orc, inp, gated=False, rows=None, scaled=True, what=""):
    N = inp["N"]
    g = inp["gate"] if gated else None
    T = inp["q"].shape[1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    out = run_f16(cuda_lib, inp, gated, scaled)[:, rows]
    qs = orc.qscale(inp["q"], N, inp["c_h"], g) if scaled else inp["q"]
    exact = orc.attention_exact(qs, inp["k"], inp["v"], rows=rows)
    return check_f16(out, exact, f16_bound(qs, inp["k"], inp["v"], rows, exact), what)


@pytest.mark.parametrize("B,N,M,H", [(1, 1024, 128, 4), (2, 1000, 77, 3), (1, 1, 5, 2), (1, 300, 0, 1),
                                     (1, 129, 300, 5), (3, 257, 1, 2)])
def test_f16_small_full_parity(cuda_lib, orc, B, N, M, H):
    inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=N, n_query=M, heads=H, batch=B)
    layer_case(cuda_lib, orc, inp, what=f"f16 B{B} N{N} M{M} H{H}")


def test_f16_gated_head_factors(cuda_lib, orc):
    inp = make_inputs(WORKLOADS["final_n8k_m1k_h8_gated"], n_ctx=2048, n_query=200)
    layer_case(cuda_lib, orc, inp, gated=True, what="f16 gated N2048 M200 H8")


def test_f16_without_query_scaling(cuda_lib, orc):
    inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=700, n_query=50, heads=3)
    layer_case(cuda_lib, orc, inp, scaled=False, what="f16 plain N700 M50 H3")


def test_f16_max_heads(cuda_lib, orc):
    inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=200, n_query=30, heads=128)
    layer_case(cuda_lib, orc, inp, what="f16 H128")


def test_f16_full_size_8k_sampled(cuda_lib, orc):
    """The full normal-precision workload (8,192 context rows, 1,024 queries, 8 heads, gated)."""
    w = WORKLOADS["final_n8k_m1k_h8_gated"]
    inp = make_inputs(w)
    T = w.n_ctx + w.n_query
    rows = np.unique(np.concatenate([np.arange(0, T, 61), [1, 127, 128, 255, 256, T - 129, T - 2, T - 1]]))
    layer_case(cuda_lib, orc, inp, gated=True, rows=rows, what="f16 N8192 M1024 H8 gated (sampled)")


def test_f16_long_context_sampled(cuda_lib, orc):
    """A context far past the rule's switch still runs on this path (the final layer)."""
    inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=32768 + 77, n_query=1000, heads=2)
    T = inp["q"].shape[1]
    rows = np.unique(np.concatenate([np.arange(3, T, 509), [0, T - 1]]))
    layer_case(cuda_lib, orc, inp, gated=True, rows=rows, what="f16 N32845 M1000 H2 gated (sampled)")


def test_precision_rule_dispatch(cuda_lib):
    """icl_layer takes the fp16 kernel up to 8,192 context rows and for the final layer, FP8 above."""
    for N, final, fp8 in ((8192, False, False), (8193, False, True), (8193, True, False)):
        inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=N, n_query=64, heads=2)
        q, k, v, c_h = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["c_h"])
        got = host(cuda_lib.icl_layer(q, k, v, N, c_h, final_layer=final))
        want = host(cuda_lib.icl_attention(q, k, v, N, c_h) if fp8 else cuda_lib.icl_attention_f16(q, k, v, N, c_h))
        assert np.array_equal(got.view(np.uint16), want.view(np.uint16)), (N, final)
    inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=100, n_query=4, heads=2)
    with pytest.raises(ValueError):
        cuda_lib.icl_layer(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), 100, dev(inp["c_h"]),
                           cache=cuda_lib.FP8Cache(1, 100, 2, "cuda"))


def test_f16_gate_needs_query_scaling(cuda_lib):
    inp = make_inputs(WORKLOADS["final_n8k_m1k_h8_gated"], n_ctx=64, n_query=4, heads=8)
    with pytest.raises(cuda_lib.SdmError) as e:
        cuda_lib.icl_attention_f16(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), 64, None, dev(inp["gate"]))
    assert e.value.status == 1
