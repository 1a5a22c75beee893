"""Boundary behaviour on a GPU: misuse comes back as status codes, nothing faults."""
import ctypes

import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200 import binding
from parity import dev

pytestmark = pytest.mark.gpu


def _small(cuda_lib):
    rng = np.random.default_rng(0)
    q = dev(rng.standard_normal((1, 300, 2, 64)).astype(np.float16))
    k = dev(rng.standard_normal((1, 256, 2, 64)).astype(np.float16))
    c = dev(np.ones(2, np.float32))
    return q, k, c


def test_host_pointer_is_rejected(cuda_lib):
    q, k, c = _small(cuda_lib)
    L = binding.lib()
    host_buf = np.zeros(300 * 2 * 64, np.float16)
    st = L.sdm_qscale_fused(ctypes.c_void_p(host_buf.ctypes.data), ctypes.c_void_p(q.data_ptr()), 1, 300, 2, 64, 10,
                            ctypes.c_void_p(c.data_ptr()), None, None)
    assert st == 4  # SDM_ERR_DEVICE_MISMATCH


def test_cache_misuse(cuda_lib):
    q, k, c = _small(cuda_lib)
    cache = cuda_lib.FP8Cache(1, 256, 2, "cuda")
    with pytest.raises(binding.SdmError) as e:                      # not fitted yet
        cuda_lib.cached_attention(q[:, :10].contiguous(), cache, c)
    assert e.value.status == 5
    cuda_lib.icl_attention(q, k, k, 256, c, cache=cache)
    q3 = torch.zeros((1, 10, 3, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(binding.SdmError) as e:                      # heads differ
        cuda_lib.cached_attention(q3, cache, torch.ones(3, device="cuda"))
    assert e.value.status == 5
    other = cuda_lib.FP8Cache(1, 128, 2, "cuda")
    with pytest.raises(binding.SdmError) as e:                      # context length differs
        cuda_lib.icl_attention(q, k, k, 256, c, cache=other)
    assert e.value.status == 5


def test_small_workspace(cuda_lib):
    q, k, c = _small(cuda_lib)
    ws = cuda_lib.new_workspace(1024, "cuda")
    with pytest.raises(binding.SdmError) as e:
        cuda_lib.icl_attention(q, k, k, 256, c, ws=ws)
    assert e.value.status == 3
    st, flags = cuda_lib.sync_status(ws)
    assert st == 0 and flags == 0


def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    """A wait that can never complete gives up after its cycle limit: the error
    word says so, sdm_sync_status returns SDM_ERR_TIMEOUT, the word is cleared,
    and the next call on the same context works."""
    ws = cuda_lib.new_workspace(256, "cuda")
    binding.selftest_wait_timeout(ws, limit_cycles=2_000_000)
    st, flags = cuda_lib.sync_status(ws)
    assert st == 6 and flags == 1 << 7
    assert cuda_lib.sync_status(ws) == (0, 0)
    q, k, c = _small(cuda_lib)
    out = cuda_lib.icl_attention(q, k, k, 256, c)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    L = binding.lib()
    assert L.sdm_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 10, None) == 1   # limit too small
