"""The workspace-free context quantisation entry point, through the C ABI.

It serves callers that cannot allocate device memory for the library (paths
that must not call cudaMalloc, plugins whose framework owns all device memory):
its amax scratch is a fixed array inside the library.  Its results must equal
those of sdm_fp8_quantize_context and the oracle's context scales and e4m3
codes bit for bit (FP8 codes and scales are compared exactly, as everywhere
else), on two calls in a row -- the second with a smaller amax than the first,
so stale scratch would show -- and sizes past the array's limit must be
refused before any work is enqueued.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200 import binding

pytestmark = pytest.mark.gpu


def _inputs(scale, seed=0, B=2, N=1000, M=77, H=3):
    rng = np.random.default_rng(seed)
    mk = lambda rows: torch.from_numpy((rng.standard_normal((B, rows, H, 64)) * scale).astype(np.float16)).cuda()
    return mk(N + M), mk(N), mk(N)


def _noalloc_call(L, q, k, v, N):
    B, T, H, d = q.shape
    cache = binding.FP8Cache(B, N, H, "cuda")
    q8 = torch.empty((B, H, T, d), dtype=torch.uint8, device="cuda")
    st = L.sdm_fp8_quantize_context_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                            ctypes.c_void_p(v.data_ptr()), B, N, T - N, H, d,
                                            ctypes.c_void_p(q8.data_ptr()), ctypes.byref(cache.struct),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, binding.STATUS_NAMES.get(st, st)
    return q8, cache


def test_noalloc_matches_workspace_entry_point_twice(cuda_lib, orc):
    L = binding.lib()
    N = 1000
    for scale in (4.0, 0.5):          # second call: smaller amax than the first
        q, k, v = _inputs(scale)
        q8_ref, c_ref = cuda_lib.fp8_quantize_context(q, k, v, N)
        q8, c = _noalloc_call(L, q, k, v, N)
        torch.cuda.synchronize()
        assert c.struct.filled == 1
        assert torch.equal(c.scales, c_ref.scales)
        assert torch.equal(q8, q8_ref)
        assert torch.equal(c.k8, c_ref.k8)
        assert torch.equal(c.v8t, c_ref.v8t)
        # and against the oracle: context-only scales, then the e4m3 codes
        qn, kn, vn = (x.cpu().numpy() for x in (q, k, v))
        s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qn, kn, vn))
        sc = c.scales.cpu().numpy()
        assert (sc[0] == s_q).all() and (sc[1] == s_k).all() and (sc[2] == s_v).all()
        assert (q8.cpu().numpy() == orc.quantize(qn, s_q)).all()
        assert (c.k8.cpu().numpy() == orc.quantize(kn, s_k)).all()
        assert (c.v8t.cpu().numpy()[..., :N] == orc.quantize(vn, s_v).transpose(0, 1, 3, 2)).all()


def test_noalloc_rejects_sizes_past_its_array(cuda_lib):
    L = binding.lib()
    B, H = 33, 128                     # B*H = 4224 > 4096
    assert B * H > binding.NOALLOC_MAX_BATCH_HEADS
    st = L.sdm_fp8_quantize_context_noalloc(None, None, None, B, 10, 0, H, 64, None, None, None)
    assert st == 2                     # SDM_ERR_UNSUPPORTED, nothing enqueued
