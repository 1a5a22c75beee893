"""The C-ABI library builds, loads and exports every symbol include/sdm_fp8.h
declares; argument errors come back as status codes before any CUDA work
(no GPU needed)."""
import ctypes
import os
import re

import pytest
import torch

from fp8_quant_logscale_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdm_fp8.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return binding.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sdm_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_layer_calls():
    syms = declared_symbols()
    for name in ("sdm_qscale_fused", "sdm_fp8_quantize_context", "sdm_icl_attention", "sdm_cached_attention"):
        assert name in syms


def test_every_declared_symbol_is_exported(L):
    syms = declared_symbols()
    assert set(syms) == set(binding.EXPORTS)
    for name in syms:
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in binding.STATUS_NAMES.items():
        assert L.sdm_status_string(code).decode().startswith(name)
    assert L.sdm_version() == 101


def test_cache_layout_and_workspace_sizes(L):
    kb, vb, sb, ld = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int64()
    st = L.sdm_cache_layout(2, 1000, 3, 64, ctypes.byref(kb), ctypes.byref(vb), ctypes.byref(sb), ctypes.byref(ld))
    assert st == 0 and ld.value == 1024
    assert kb.value == 2 * 3 * 1000 * 64 and vb.value == 2 * 3 * 64 * 1024 and sb.value == (3 * 2 * 3 + 2 * 2) * 4  # scales + ragged meta
    assert L.sdm_cache_layout(1, 1000, 3, 32, None, None, None, None) == 2       # d != 64
    assert L.sdm_cache_layout(1, 0, 3, 64, None, None, None, None) == 1          # N < 1
    assert L.sdm_cache_layout(1, 10, 129, 64, None, None, None, None) == 2       # too many heads
    w_icl = binding.workspace_size(binding.OP_ICL_ATTENTION, 1, 16384, 1024, 8, keep_cache=True)
    w_icl_nc = binding.workspace_size(binding.OP_ICL_ATTENTION, 1, 16384, 1024, 8, keep_cache=False)
    assert w_icl >= 8 * 17408 * 64 and w_icl_nc >= w_icl + 2 * 8 * 16384 * 64
    w_c = binding.workspace_size(binding.OP_CACHED_ATTENTION, 1, 524288, 1024, 8)
    assert w_c >= 32 * 8 * 1024 * 66 * 4                                           # 32 split-KV partials
    assert L.sdm_workspace_size(0, 1, 100, 0, 8, 32, 1) == 0
    assert L.sdm_workspace_size(7, 1, 100, 0, 8, 64, 1) == 0


def test_shape_errors_before_any_cuda_call(L):
    assert L.sdm_qscale_fused(None, None, 1, 10, 4, 32, 10, None, None, None) == 2
    assert L.sdm_qscale_fused(None, None, 0, 10, 4, 64, 10, None, None, None) == 1
    assert L.sdm_icl_attention(None, None, None, 1, 0, 5, 4, 64, None, None, None, None, None, 0, None) == 1
    assert L.sdm_icl_attention(None, None, None, 1, 10, 5, 4, 48, None, None, None, None, None, 0, None) == 2
    assert L.sdm_cached_attention(None, 1, 5, 4, 64, None, None, None, None, None, 0, None) == 1
    assert L.sdm_fp8_attention(None, 1, 5, None, None, 0, None, 0, None) == 1
    assert L.sdm_sync_status(None, None, None) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_reports_cuda_error(L):
    # valid shapes, no GPU: the device query fails and nothing is launched
    assert L.sdm_qscale_fused(None, None, 1, 10, 4, 64, 10, None, None, None) == 7


def test_split_length_rule_matches_the_oracle(L, orc):
    """Cached prediction's chunk length is a function of N alone, the same on both sides."""
    for n in [1, 100, 1024, 4096, 4097, 16384, 20000, 131072, 131073, 524288, 1 << 22, 1 << 26]:
        assert L.sdm_split_keys(n) == orc.split_keys(n), n
    assert L.sdm_split_keys(524288) == 16384 and L.sdm_split_keys(16384) == 1024
    assert L.sdm_split_keys(0) == 0


def test_precision_rule(L):
    # FP8 only on a non-final ICL layer with more than 8,192 unmasked context rows
    assert binding.FP8_MIN_CONTEXT == 8192
    assert not binding.fp8_eligible(8192) and binding.fp8_eligible(8193)
    assert not binding.fp8_eligible(1 << 20, final_layer=True)
    assert not binding.fp8_eligible(0) and not binding.fp8_eligible(-5)
    for n in (1, 1024, 8191, 8192, 8193, 16384, 524288):
        for final in (0, 1):
            assert L.sdm_fp8_eligible(n, final) == int(final == 0 and n > 8192)


def test_f16_workspace_and_shape_errors(L):
    # q' [B][T][H][64] fp16 plus V^T [B][H][64][round_up(N, 128)] fp16
    w = binding.workspace_size(binding.OP_ICL_ATTENTION_F16, 2, 1000, 24, 3)
    assert w >= 256 + 2 * 1024 * 3 * 64 * 2 + 2 * 3 * 64 * 1024 * 2
    assert binding.workspace_size(binding.OP_ICL_ATTENTION_F16, 1, 0, 8, 4) == 0
    assert L.sdm_icl_attention_f16(None, None, None, 1, 0, 5, 4, 64, None, None, None, None, 0, None) == 1
    assert L.sdm_icl_attention_f16(None, None, None, 1, 10, 5, 4, 48, None, None, None, None, 0, None) == 2
    assert L.sdm_icl_attention_f16(None, None, None, 1, 10, 5, 200, 64, None, None, None, None, 0, None) == 2


def test_ragged_argument_errors(L):
    import ctypes as C
    lens = lambda *x: (C.c_int64 * len(x))(*x)
    f = L.sdm_icl_attention_ragged
    assert f(None, None, None, 2, 100, 5, 4, 64, None, None, None, None, None, None, 0, None) == 1   # no ctx_len
    assert f(None, None, None, 2, 100, 5, 4, 64, lens(100, 0), None, None, None, None, None, 0, None) == 1
    assert f(None, None, None, 2, 100, 5, 4, 64, lens(101, 50), None, None, None, None, None, 0, None) == 1
    g = L.sdm_icl_attention_f16_ragged
    assert g(None, None, None, 2, 100, 5, 4, 64, None, None, None, None, None, 0, None) == 1
    assert g(None, None, None, 2, 100, 5, 4, 64, lens(-3, 7), None, None, None, None, 0, None) == 1
    if not torch.cuda.is_available():  # valid lengths get past the host checks to the device query
        assert f(None, None, None, 2, 100, 5, 4, 64, lens(100, 1), None, None, None, None, None, 0, None) == 7


def test_prefill_argument_errors(L):
    import ctypes as C
    ip = lambda *x: (C.c_int64 * len(x))(*x)
    f = L.sdm_gqa_prefill
    assert f(None, None, None, None, None, 1, 16, 4, 128, 1, None, None, 0, None) == 1      # no indptr
    assert f(None, None, None, ip(0, 5), ip(0, 10), 1, 16, 4, 64, 1, None, None, 0, None) == 2   # head dim
    assert f(None, None, None, ip(0, 5), ip(0, 10), 1, 16, 3, 128, 1, None, None, 0, None) == 1  # 16 % 3
    assert f(None, None, None, ip(0, 5), ip(0, 10), 1, 64, 2, 128, 1, None, None, 0, None) == 2  # group 32
    assert f(None, None, None, ip(0, 5), ip(0, 4), 1, 16, 4, 128, 1, None, None, 0, None) == 1   # kv < q, causal
    assert f(None, None, None, ip(0, 5), ip(0, 0), 1, 16, 4, 128, 0, None, None, 0, None) == 1   # no keys
    assert f(None, None, None, ip(1, 5), ip(0, 10), 1, 16, 4, 128, 1, None, None, 0, None) == 1  # offsets from 0
    assert f(None, None, None, ip(0, 0), ip(0, 0), 1, 16, 4, 128, 1, None, None, 0, None) == 0   # nothing to do
    # the error word only: a query tile's key shares are combined on chip (cluster shared memory)
    assert binding.gqa_prefill_workspace_size([0, 64], [0, 5000], 16, 4) == 256
    assert binding.gqa_prefill_workspace_size([0, 64], [0, 10], 16, 4) == 0          # kv < q, causal
    assert binding.gqa_prefill_workspace_size([0, 64], [0, 10], 16, 4, causal=False) > 0
