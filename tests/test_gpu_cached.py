"""GPU parity of step 4 (cached prediction with split-KV) against the oracle, and
bitwise equality of the cached outputs across query batch splits."""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import AMB, dev, gate, host

pytestmark = pytest.mark.gpu


def _fit(cuda_lib, inp):
    B, N, H = inp["B"], inp["N"], inp["H"]
    cache = cuda_lib.FP8Cache(B, N, H, "cuda")
    cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache)
    return cache


def _oracle_cached(orc, inp, queries, rows=None):
    N = inp["N"]
    qs = orc.qscale(inp["q"], N, inp["c_h"])
    s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qs, inp["k"], inp["v"]))
    k8, v8 = orc.quantize(inp["k"], s_k), orc.quantize(inp["v"], s_v)
    qq = orc.quantize(orc.qscale(queries, N, inp["c_h"]), s_q)
    return orc.attention(qq, k8, v8, s_q, s_k, s_v, rows=rows, split=orc.split_keys(N), **AMB)


@pytest.mark.parametrize("N,M,H", [(20000, 300, 3), (16384, 64, 8), (1000, 1, 2), (33000, 129, 4)])
def test_cached_parity(cuda_lib, orc, N, M, H):
    inp = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=N, n_query=M, heads=H)
    cache = _fit(cuda_lib, inp)
    out = cuda_lib.cached_attention(dev(inp["queries"]), cache, dev(inp["c_h"]))
    torch.cuda.synchronize()
    _, o, allow = _oracle_cached(orc, inp, inp["queries"])
    print(f"\ncached N{N} M{M} H{H}:", gate(out, o, allow, "cached"))


def _split_equal(cuda_lib, cache, queries, c_h):
    full = host(cuda_lib.cached_attention(queries, cache, c_h))
    for part in (64, 1):
        pieces = [host(cuda_lib.cached_attention(queries[:, i:i + part].contiguous(), cache, c_h))
                  for i in range(0, queries.shape[1], part)]
        got = np.concatenate(pieces, axis=1)
        assert (got.view(np.uint16) == full.view(np.uint16)).all(), f"batch split {part} differs"
    return full


def test_batch_split_invariance_small(cuda_lib):
    inp = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=40000, n_query=1024, heads=2)
    cache = _fit(cuda_lib, inp)
    _split_equal(cuda_lib, cache, dev(inp["queries"]), dev(inp["c_h"]))


def test_cached_512k_full_size(cuda_lib, orc):
    """The cached-prediction workload: 1,024 queries against a 524,288-row FP8 cache,
    bitwise equal across batch splits 1/64/1024, every query checked against the oracle."""
    w = WORKLOADS["cached_n512k_m1k_h8"]
    inp = make_inputs(w)
    cache = _fit(cuda_lib, inp)
    full = _split_equal(cuda_lib, cache, dev(inp["queries"]), dev(inp["c_h"]))
    _, o, allow = _oracle_cached(orc, inp, inp["queries"])
    print("\ncached 512K:", gate(full, o, allow, "cached 512K"))


def test_cached_batch2_gated_queries(cuda_lib, orc):
    """B = 2 (per-(b, h) scales) and GatedLogScale on the prediction queries."""
    B, N, M, H = 2, 17000, 40, 3
    inp = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=N, n_query=M, heads=H, batch=B)
    cache = _fit(cuda_lib, inp)
    rng = np.random.default_rng(7)
    g_q = (rng.standard_normal((B, M, H)) * 1.5).astype(np.float16)
    out = cuda_lib.cached_attention(dev(inp["queries"]), cache, dev(inp["c_h"]), dev(g_q))
    torch.cuda.synchronize()
    qs = orc.qscale(inp["q"], N, inp["c_h"])
    s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qs, inp["k"], inp["v"]))
    qq = orc.quantize(orc.qscale(inp["queries"], N, inp["c_h"], g_q), s_q)
    _, o, allow = orc.attention(qq, orc.quantize(inp["k"], s_k), orc.quantize(inp["v"], s_v), s_q, s_k, s_v,
                                split=orc.split_keys(N), **AMB)
    print("\ncached B2 gated:", gate(out, o, allow, "cached B2 gated"))
