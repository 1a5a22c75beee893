"""GPU parity of batched estimators with ragged (padded) contexts against the
oracle's per-estimator composition (layer_ragged): FP8 codes and scales bit for
bit, outputs within the layer's gates, padding rows exactly zero whatever they
hold (NaN and infinities included), cached prediction against a ragged cache,
and the normal-precision path."""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import AMB, dev, gate, host
from test_gpu_attention_f16 import check_f16, f16_bound

pytestmark = pytest.mark.gpu
W = WORKLOADS["ragged_b16_n16k_m1k_h8"]


def poison_padding(inp):
    """Padding rows get NaN / huge / infinite values: none may reach a result."""
    N = inp["N"]
    q, k, v = inp["q"].copy(), inp["k"].copy(), inp["v"].copy()
    for b, n in enumerate(inp["ctx_len"]):
        q[b, n:N] = np.float16(np.nan)
        k[b, n:] = np.float16(np.nan)
        v[b, n:] = np.float16(np.inf)
    return dict(inp, q=q, k=k, v=v)


def fit_ragged(cuda_lib, inp, gated=False):
    B, N, M, H = inp["B"], inp["N"], inp["M"], inp["H"]
    cache = cuda_lib.FP8Cache(B, N, H, "cuda")
    ws = cuda_lib.new_workspace(cuda_lib.workspace_size(1, B, N, M, H, keep_cache=True), "cuda")
    out = cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]),
                                 dev(inp["gate"] if gated else None), cache=cache, ws=ws, ctx_len=inp["ctx_len"])
    st, flags = cuda_lib.sync_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    return host(out), cache


@pytest.mark.parametrize("B,N,M,H,lens", [(3, 300, 20, 2, None), (2, 257, 9, 3, [129, 257]),
                                          (4, 1000, 130, 2, [1, 1000, 128, 129]), (2, 2048, 300, 4, None)])
def test_ragged_fit_parity(cuda_lib, orc, B, N, M, H, lens):
    inp = make_inputs(W, n_ctx=N, n_query=M, heads=H, batch=B)
    if lens is not None:
        inp["ctx_len"] = np.array(lens, np.int64)
    inp = poison_padding(inp)
    out, cache = fit_ragged(cuda_lib, inp)
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], inp["ctx_len"], inp["c_h"], **AMB)
    sc = host(cache.scales)
    assert (sc[0] == r["s_q"]).all() and (sc[1] == r["s_k"]).all() and (sc[2] == r["s_v"]).all()
    assert (host(cache.k8) == r["k8"]).all()
    assert (host(cache.v8t)[..., :N] == r["v8"].transpose(0, 1, 3, 2)).all()
    assert not host(cache.v8t)[..., N:].any()
    assert cache.ragged and cache.ctx_len() == [int(x) for x in inp["ctx_len"]]
    for b, n in enumerate(inp["ctx_len"]):
        assert not out[b, n:N].view(np.uint16).any(), f"padding rows of batch {b} not zero"
    stats = gate(out, r["out"], r["allow"], f"ragged B{B} N{N} M{M} H{H}")
    print(f"\nragged B{B} N{N} M{M} H{H} lens {list(inp['ctx_len'])}: {stats}")


def test_ragged_gated(cuda_lib, orc):
    inp = make_inputs(W, n_ctx=700, n_query=40, heads=2, batch=3)
    inp["gate"] = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=700, n_query=40, heads=2,
                              batch=3)["gate"]
    out, cache = fit_ragged(cuda_lib, inp, gated=True)
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], inp["ctx_len"], inp["c_h"], inp["gate"], **AMB)
    assert (host(cache.scales)[0] == r["s_q"]).all()
    gate(out, r["out"], r["allow"], "ragged gated")


def test_ragged_full_lengths_equal_the_uniform_call(cuda_lib):
    inp = make_inputs(W, n_ctx=900, n_query=64, heads=2, batch=2)
    N = inp["N"]
    inp["ctx_len"] = np.array([N, N])
    out_r, _ = fit_ragged(cuda_lib, inp)
    out_u = host(cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"])))
    assert np.array_equal(out_r.view(np.uint16), out_u.view(np.uint16))


def test_cached_prediction_against_a_ragged_cache(cuda_lib, orc):
    """Queries of batch b: scaled with n = n_b, quantised with its s_q, keys [0, n_b),
    split-KV in chunks of split_keys(N) (chunks past n_b are empty)."""
    B, N, M, H = 3, 3000, 64, 2
    inp = make_inputs(W, n_ctx=N, n_query=0, heads=H, batch=B)
    inp["ctx_len"] = np.array([900, 3000, 1025], np.int64)
    inp = poison_padding(inp)
    _, cache = fit_ragged(cuda_lib, inp)
    queries = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=8, n_query=M, heads=H, batch=B)["queries"]
    pred = host(cuda_lib.cached_attention(dev(queries), cache, dev(inp["c_h"])))
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], inp["ctx_len"], inp["c_h"])
    L = orc.split_keys(N)
    for b, n in enumerate(inp["ctx_len"]):
        qs = orc.qscale(queries[b:b + 1], int(n), inp["c_h"])
        q8 = orc.quantize(qs, r["s_q"][b:b + 1])
        k8 = np.ascontiguousarray(r["k8"][b:b + 1, :, :n])
        v8 = np.ascontiguousarray(r["v8"][b:b + 1, :, :n])
        o16, o, allow = orc.attention(q8, k8, v8, r["s_q"][b:b + 1], r["s_k"][b:b + 1], r["s_v"][b:b + 1],
                                      split=L, **AMB)
        gate(pred[b:b + 1], o, allow, f"cached ragged batch {b} n_b={n}")
    # batch invariance: one query at a time gives the same bits
    one = host(cuda_lib.cached_attention(dev(queries[:, 5:6].copy()), cache, dev(inp["c_h"])))
    assert np.array_equal(one.view(np.uint16), pred[:, 5:6].view(np.uint16))


def test_f16_ragged(cuda_lib, orc):
    inp = poison_padding(make_inputs(W, n_ctx=1000, n_query=77, heads=3, batch=3))
    B, N, M, H = inp["B"], inp["N"], inp["M"], inp["H"]
    out = host(cuda_lib.icl_attention_f16(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]),
                                          ctx_len=inp["ctx_len"]))
    for b, n in enumerate(inp["ctx_len"]):
        assert not out[b, n:N].view(np.uint16).any()
        rows = np.r_[0:n, N:N + M]
        qs = orc.qscale(np.ascontiguousarray(inp["q"][b:b + 1, rows]), int(n), inp["c_h"])
        k = np.ascontiguousarray(inp["k"][b:b + 1, :n])
        v = np.ascontiguousarray(inp["v"][b:b + 1, :n])
        exact = orc.attention_exact(qs, k, v)
        all_rows = np.arange(rows.size)
        check_f16(out[b:b + 1, rows], exact, f16_bound(qs, k, v, all_rows, exact), f"f16 ragged batch {b} n_b={n}")


def test_full_size_ragged_workload_sampled(cuda_lib, orc):
    """16 estimators padded to 16,384 rows: padding rows zero, two estimators' sampled
    rows against the oracle's layer on that estimator alone."""
    inp = make_inputs(W)
    B, N, M, H = inp["B"], inp["N"], inp["M"], inp["H"]
    out, cache = fit_ragged(cuda_lib, inp)
    lens = inp["ctx_len"]
    for b, n in enumerate(lens):
        assert not out[b, n:N].view(np.uint16).any()
    sc = host(cache.scales)
    for b in (int(np.argmin(lens)), int(np.argmax(lens))):
        n = int(lens[b])
        rows_b = np.r_[0:n, N:N + M]
        sel = np.unique(np.r_[np.arange(0, rows_b.size, 97), [n - 1, n, rows_b.size - 1]]).astype(np.int64)
        r = orc.layer(np.ascontiguousarray(inp["q"][b:b + 1, rows_b]), np.ascontiguousarray(inp["k"][b:b + 1, :n]),
                      np.ascontiguousarray(inp["v"][b:b + 1, :n]), n, inp["c_h"], rows=sel, **AMB)
        assert (sc[0][b] == r["s_q"][0]).all() and (sc[1][b] == r["s_k"][0]).all()
        gate(out[b:b + 1, rows_b[sel]], r["out"], r["allow"], f"full ragged batch {b} n_b={n}")


def test_ragged_long_context_decoupled_issue(cuda_lib, orc):
    """At 262,144 keys and more the one-call layer issues each query tile's MMAs from its
    own warp: a ragged batch there (a ragged last key tile, padding rows, CTAs whose rows
    are all padding) against the oracle's layer on each estimator alone, sampled rows."""
    B, N, M, H = 2, 262144, 64, 2
    inp = make_inputs(W, n_ctx=N, n_query=M, heads=H, batch=B)
    inp["ctx_len"] = np.array([N, 150017], np.int64)
    inp = poison_padding(inp)
    out, cache = fit_ragged(cuda_lib, inp)
    sc = host(cache.scales)
    for b, n in enumerate(inp["ctx_len"]):
        n = int(n)
        assert not out[b, n:N].view(np.uint16).any(), f"padding rows of batch {b} not zero"
        rows_b = np.r_[0:n, N:N + M]
        sel = np.unique(np.r_[np.arange(0, n, n // 40), [1, n - 1], np.arange(n, n + M)]).astype(np.int64)
        r = orc.layer(np.ascontiguousarray(inp["q"][b:b + 1, rows_b]), np.ascontiguousarray(inp["k"][b:b + 1, :n]),
                      np.ascontiguousarray(inp["v"][b:b + 1, :n]), n, inp["c_h"], rows=sel, **AMB)
        assert (sc[0][b] == r["s_q"][0]).all() and (sc[1][b] == r["s_k"][0]).all() and (sc[2][b] == r["s_v"][0]).all()
        stats = gate(out[b:b + 1, rows_b[sel]], r["out"], r["allow"], f"long ragged batch {b} n_b={n}")
        print(f"\nlong ragged batch {b} n_b={n}: {stats}")


def test_precision_rule_uses_the_smallest_estimator(cuda_lib):
    inp = make_inputs(W, n_ctx=9000, n_query=16, heads=2, batch=2)
    N = inp["N"]
    q, k, v, c_h = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["c_h"])
    for lens, fp8 in (([9000, 8193], True), ([9000, 8192], False)):
        got = host(cuda_lib.icl_layer(q, k, v, N, c_h, ctx_len=lens))
        want = host(cuda_lib.icl_attention(q, k, v, N, c_h, ctx_len=lens) if fp8
                    else cuda_lib.icl_attention_f16(q, k, v, N, c_h, ctx_len=lens))
        assert np.array_equal(got.view(np.uint16), want.view(np.uint16)), lens
