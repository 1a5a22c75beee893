"""Cached prediction from a cache held in page-locked host memory
(sdm_cached_attention_offload): chunk by chunk through two device staging slots,
it must give the same bits as sdm_cached_attention on the device-resident cache
(the same split-KV chunks, the same fixed-order combine), with and without a
separate copy stream, for uniform and ragged caches, and at full size -- and,
on its own, match the oracle's chunked attention within the layer's gates (a
seeded sample of queries at full size, every query of a ragged cache)."""
import ctypes

import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import AMB, dev, gate, host

pytestmark = pytest.mark.gpu


def fitted(cuda_lib, N, H, B=1, ctx_len=None, wname="cached_n512k_m1k_h8"):
    inp = make_inputs(WORKLOADS[wname], n_ctx=N, n_query=0, heads=H, batch=B)
    cache = cuda_lib.FP8Cache(B, N, H, "cuda")
    cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache,
                           ctx_len=ctx_len)
    return inp, cache


def queries(H, M, B=1):
    return make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=8, n_query=M, heads=H, batch=B)["queries"]


def same(a, b):
    return np.array_equal(host(a).view(np.uint16), host(b).view(np.uint16))


@pytest.mark.parametrize("N,M", [(40000, 1), (40000, 64), (40000, 1000), (300, 17), (1024, 5), (1025, 130)])
def test_offload_equals_resident(cuda_lib, N, M):
    H = 2
    inp, cache = fitted(cuda_lib, N, H)
    off = cache.offload()
    assert off.k8.is_pinned() and off.v8t.is_pinned()
    q, c_h = dev(queries(H, M)), dev(inp["c_h"])
    want = cuda_lib.cached_attention(q, cache, c_h)
    got = cuda_lib.cached_attention_offload(q, off, c_h)                       # side copy stream
    one = cuda_lib.cached_attention_offload(q, off, c_h, copy_stream=torch.cuda.current_stream())
    ws = cuda_lib.new_workspace(cuda_lib.workspace_size(cuda_lib.OP_CACHED_ATTENTION_OFFLOAD, 1, N, M, H), "cuda")
    again = cuda_lib.cached_attention_offload(q, off, c_h, ws=ws)
    again2 = cuda_lib.cached_attention_offload(q, off, c_h, ws=ws)            # reused workspace and slots
    torch.cuda.synchronize()
    assert cuda_lib.sync_status(ws) == (0, 0)
    for x in (got, one, again, again2):
        assert same(x, want)


def test_offload_gated_queries(cuda_lib):
    H, M, N = 8, 100, 20000
    inp, cache = fitted(cuda_lib, N, H)
    gate = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=8, n_query=M - 8, heads=H)["gate"]
    q, c_h, g = dev(queries(H, M)), dev(inp["c_h"]), dev(gate)
    assert same(cuda_lib.cached_attention_offload(q, cache.offload(), c_h, gate=g),
                cuda_lib.cached_attention(q, cache, c_h, gate=g))


def test_offload_ragged_cache(cuda_lib, orc):
    H, B, N, M = 2, 3, 3000, 40
    lens = [900, 3000, 1025]
    inp, cache = fitted(cuda_lib, N, H, B=B, ctx_len=lens, wname="ragged_b16_n16k_m1k_h8")
    off = cache.offload()
    qn = queries(H, M, B)
    q, c_h = dev(qn), dev(inp["c_h"])
    got = cuda_lib.cached_attention_offload(q, off, c_h)
    assert same(got, cuda_lib.cached_attention(q, cache, c_h))
    # against the oracle: estimator b is the layer on its own n_b context rows
    got = host(got)
    r = orc.layer_ragged(inp["q"], inp["k"], inp["v"], lens, inp["c_h"])
    for b, n in enumerate(lens):
        q8 = orc.quantize(orc.qscale(qn[b:b + 1], n, inp["c_h"]), r["s_q"][b:b + 1])
        _, o, allow = orc.attention(q8, np.ascontiguousarray(r["k8"][b:b + 1, :, :n]),
                                    np.ascontiguousarray(r["v8"][b:b + 1, :, :n]), r["s_q"][b:b + 1],
                                    r["s_k"][b:b + 1], r["s_v"][b:b + 1], split=orc.split_keys(N), **AMB)
        print(f"\noffload ragged batch {b} n_b={n}:", gate(got[b:b + 1], o, allow, f"offload ragged b{b}"))


def test_offload_full_size(cuda_lib, orc):
    """The 524,288-key cache (537 MB of K8 / V8^T in host memory), 1,024 queries: equal to
    the resident cache bit for bit, and a seeded sample of 256 queries (every head)
    against the oracle's chunked attention."""
    w = WORKLOADS["cached_n512k_m1k_h8"]
    inp = make_inputs(w)
    N, M, H = w.n_ctx, w.n_query, w.heads
    cache = cuda_lib.FP8Cache(1, N, H, "cuda")
    cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache)
    q, c_h = dev(inp["queries"]), dev(inp["c_h"])
    want = cuda_lib.cached_attention(q, cache, c_h)
    off = cache.offload()
    del cache
    torch.cuda.empty_cache()
    got = cuda_lib.cached_attention_offload(q, off, c_h)
    assert same(got, want)
    assert same(cuda_lib.cached_attention_offload(q[:, :1].contiguous(), off, c_h), want[:, :1])
    rows = np.sort(np.random.default_rng(5).choice(M, 256, replace=False)).astype(np.int64)
    qs = orc.qscale(inp["q"], N, inp["c_h"])
    s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qs, inp["k"], inp["v"]))
    q8 = orc.quantize(orc.qscale(inp["queries"], N, inp["c_h"]), s_q)
    _, o, allow = orc.attention(q8, orc.quantize(inp["k"], s_k), orc.quantize(inp["v"], s_v), s_q, s_k, s_v,
                                rows=rows, split=orc.split_keys(N), **AMB)
    print("\noffload 512K, 256 queries:", gate(host(got)[:, rows], o, allow, "offload 512K"))


def test_offload_rejects_pageable_memory(cuda_lib):
    H, N = 2, 2000
    inp, cache = fitted(cuda_lib, N, H)
    off = cache.offload()
    pageable_k = torch.empty(off.k8.shape, dtype=torch.uint8)   # not page-locked
    pageable_k.copy_(off.k8)
    off.struct.k8 = pageable_k.data_ptr()
    with pytest.raises(cuda_lib.SdmError) as e:
        cuda_lib.cached_attention_offload(dev(queries(H, 4)), off, dev(inp["c_h"]))
    assert e.value.status == 5
