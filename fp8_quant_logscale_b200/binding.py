"""ctypes binding of ``libsdm_fp8.so`` (the C ABI in ``include/sdm_fp8.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch supplies device memory, the current stream and dtype checks.
If the shared library is missing, every call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdm_fp8.so")

SDM_OK = 0
STATUS_NAMES = {0: "SDM_OK", 1: "SDM_ERR_INVALID_ARG", 2: "SDM_ERR_UNSUPPORTED", 3: "SDM_ERR_WORKSPACE",
                4: "SDM_ERR_DEVICE_MISMATCH", 5: "SDM_ERR_CACHE_MISMATCH", 6: "SDM_ERR_TIMEOUT",
                7: "SDM_ERR_CUDA"}
OP_QUANTIZE_CONTEXT, OP_ICL_ATTENTION, OP_CACHED_ATTENTION, OP_ICL_ATTENTION_F16 = 0, 1, 2, 3
OP_CACHED_ATTENTION_OFFLOAD = 4
OP_CACHED_PARTIALS = 5
FP8_MIN_CONTEXT = 8192
KV_TILE = 128
HEAD_DIM = 64

# Every symbol the header declares (checked by the ABI tests).
EXPORTS = ("sdm_status_string", "sdm_version", "sdm_split_keys", "sdm_cache_layout", "sdm_workspace_size", "sdm_qscale_fused",
           "sdm_fp8_quantize_context", "sdm_fp8_quantize_context_noalloc", "sdm_fp8_attention", "sdm_icl_attention",
           "sdm_cached_attention", "sdm_fp8_eligible", "sdm_icl_attention_f16", "sdm_icl_attention_ragged",
           "sdm_icl_attention_f16_ragged", "sdm_cached_attention_offload", "sdm_gqa_prefill",
           "sdm_gqa_prefill_workspace_size", "sdm_sync_status",
           "sdm_selftest_wait_timeout", "sdm_context_amax", "sdm_quantize_with_scales", "sdm_cache_put_rows",
           "sdm_cached_partials", "sdm_cached_combine")
NOALLOC_MAX_BATCH_HEADS = 4096


class SdmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({_status_string(status)})")


class CacheStruct(ctypes.Structure):
    _fields_ = [("k8", ctypes.c_void_p), ("v8t", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("n_ctx", ctypes.c_int64), ("ld_v", ctypes.c_int64), ("batch", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("device", ctypes.c_int32),
                ("filled", ctypes.c_int32), ("ragged", ctypes.c_int32)]


_lib = None
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libsdm_fp8.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run fp8_quant_logscale_b200/build.py "
                               "(or __graft_entry__.build()) first; there is no CPU fallback")
        L = ctypes.CDLL(LIB_PATH)
        L.sdm_status_string.restype = ctypes.c_char_p
        L.sdm_status_string.argtypes = [ctypes.c_int]
        L.sdm_version.restype = _I32
        L.sdm_version.argtypes = []
        L.sdm_split_keys.restype = _I64
        L.sdm_split_keys.argtypes = [_I64]
        L.sdm_cache_layout.restype = ctypes.c_int
        L.sdm_cache_layout.argtypes = [_I32, _I64, _I32, _I32, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ),
                                       ctypes.POINTER(_SZ), ctypes.POINTER(_I64)]
        L.sdm_workspace_size.restype = _SZ
        L.sdm_workspace_size.argtypes = [ctypes.c_int, _I32, _I64, _I64, _I32, _I32, _I32]
        L.sdm_qscale_fused.restype = ctypes.c_int
        L.sdm_qscale_fused.argtypes = [_P, _P, _I32, _I64, _I32, _I32, _I64, _P, _P, _P]
        L.sdm_fp8_quantize_context.restype = ctypes.c_int
        L.sdm_fp8_quantize_context.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _P,
                                               ctypes.POINTER(CacheStruct), _P, _SZ, _P]
        L.sdm_fp8_quantize_context_noalloc.restype = ctypes.c_int
        L.sdm_fp8_quantize_context_noalloc.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _P,
                                                       ctypes.POINTER(CacheStruct), _P]
        L.sdm_fp8_attention.restype = ctypes.c_int
        L.sdm_fp8_attention.argtypes = [_P, _I32, _I64, ctypes.POINTER(CacheStruct), _P, _I32, _P, _SZ, _P]
        L.sdm_icl_attention.restype = ctypes.c_int
        L.sdm_icl_attention.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _P, _P, _P,
                                        ctypes.POINTER(CacheStruct), _P, _SZ, _P]
        L.sdm_cached_attention.restype = ctypes.c_int
        L.sdm_cached_attention.argtypes = [_P, _I32, _I64, _I32, _I32, ctypes.POINTER(CacheStruct), _P, _P, _P,
                                           _P, _SZ, _P]
        L.sdm_icl_attention_ragged.restype = ctypes.c_int
        L.sdm_icl_attention_ragged.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _P, _P, _P, _P,
                                               ctypes.POINTER(CacheStruct), _P, _SZ, _P]
        L.sdm_icl_attention_f16_ragged.restype = ctypes.c_int
        L.sdm_icl_attention_f16_ragged.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _P, _P, _P, _P,
                                                   _P, _SZ, _P]
        L.sdm_cached_attention_offload.restype = ctypes.c_int
        L.sdm_cached_attention_offload.argtypes = [_P, _I32, _I64, _I32, _I32, ctypes.POINTER(CacheStruct), _P, _P,
                                                   _P, _P, _SZ, _P, _P]
        L.sdm_gqa_prefill.restype = ctypes.c_int
        L.sdm_gqa_prefill.argtypes = [_P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P, _P, _SZ, _P]
        L.sdm_gqa_prefill_workspace_size.restype = _SZ
        L.sdm_gqa_prefill_workspace_size.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _I32]
        L.sdm_fp8_eligible.restype = _I32
        L.sdm_fp8_eligible.argtypes = [_I64, _I32]
        L.sdm_icl_attention_f16.restype = ctypes.c_int
        L.sdm_icl_attention_f16.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _SZ, _P]
        L.sdm_selftest_wait_timeout.restype = ctypes.c_int
        L.sdm_selftest_wait_timeout.argtypes = [_P, _I64, _P]
        L.sdm_sync_status.restype = ctypes.c_int
        L.sdm_sync_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint32)]
        L.sdm_context_amax.restype = ctypes.c_int
        L.sdm_context_amax.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _I64, _P, _P, _P, _P]
        L.sdm_quantize_with_scales.restype = ctypes.c_int
        L.sdm_quantize_with_scales.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _I64, _P, _P, _P, _P,
                                               _P, _P, _I64, _P, _I64, _P]
        L.sdm_cached_partials.restype = ctypes.c_int
        L.sdm_cached_partials.argtypes = [_P, _I32, _I64, _I32, _I32, ctypes.POINTER(CacheStruct), _P, _P, _I64,
                                          _I64, _I64, _P, _P, _P, _P, _P, _SZ, _P]
        L.sdm_cached_combine.restype = ctypes.c_int
        L.sdm_cached_combine.argtypes = [_P, _P, _I32, _I64, _I32, _I32, ctypes.POINTER(CacheStruct), _P, _P]
        L.sdm_cache_put_rows.restype = ctypes.c_int
        L.sdm_cache_put_rows.argtypes = [ctypes.POINTER(CacheStruct), _P, _I64, _P, _I64, _I64, _I64, _P]
        _lib = L
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().sdm_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - only while reporting another error
        return "?"


def _check(status: int, what: str) -> None:
    if status != SDM_OK:
        raise SdmError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _want(t: torch.Tensor, dtype: torch.dtype, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


# ------------------------------------------------------------------- sizes

def workspace_size(op: int, batch: int, n_ctx: int, n_query: int, heads: int, keep_cache: bool = True) -> int:
    return int(lib().sdm_workspace_size(op, batch, n_ctx, n_query, heads, HEAD_DIM, 1 if keep_cache else 0))


def split_keys(n_ctx: int) -> int:
    """Keys per split-KV chunk of cached prediction for an n_ctx-key context."""
    return int(lib().sdm_split_keys(int(n_ctx)))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """Zero-filled workspace (the error word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def sync_status(ws: torch.Tensor) -> tuple[int, int]:
    """(status, raw error flags) of the kernels that used `ws`; synchronises the current stream."""
    flags = ctypes.c_uint32(0)
    st = lib().sdm_sync_status(_ptr(ws), _stream(ws.device), ctypes.byref(flags))
    return int(st), int(flags.value)


def selftest_wait_timeout(ws: torch.Tensor, limit_cycles: int = 1_000_000) -> None:
    """Enqueue the bounded-wait self-test on `ws` (see sdm_selftest_wait_timeout)."""
    with torch.cuda.device(ws.device):
        _check(lib().sdm_selftest_wait_timeout(_ptr(ws), int(limit_cycles), _stream(ws.device)),
               "sdm_selftest_wait_timeout")


def _ctx_len_array(ctx_len, batch: int):
    """Host int64 array of the per-batch context lengths (ragged batches)."""
    lens = [int(x) for x in ctx_len]
    if len(lens) != batch:
        raise ValueError(f"ctx_len has {len(lens)} entries for batch {batch}")
    return (ctypes.c_int64 * batch)(*lens)


class FP8Cache:
    """Caller-owned FP8 K/V cache (k8 [B,H,N,64], v8t [B,H,64,ld_v], scales block: scales [3,B,H]
    followed by the per-batch context lengths of a ragged fit)."""

    def __init__(self, batch: int, n_ctx: int, heads: int, device):
        kb, vb, sb, ld = _SZ(), _SZ(), _SZ(), _I64()
        _check(lib().sdm_cache_layout(batch, n_ctx, heads, HEAD_DIM, ctypes.byref(kb), ctypes.byref(vb),
                                      ctypes.byref(sb), ctypes.byref(ld)), "sdm_cache_layout")
        device = torch.device(device)
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.k8 = torch.empty((batch, heads, n_ctx, HEAD_DIM), dtype=torch.uint8, device=device)
        self.v8t = torch.empty((batch, heads, HEAD_DIM, ld.value), dtype=torch.uint8, device=device)
        self.block = torch.zeros(sb.value // 4, dtype=torch.float32, device=device)
        self.scales = self.block[:3 * batch * heads].view(3, batch, heads)
        assert self.k8.numel() == kb.value and self.v8t.numel() == vb.value and self.block.numel() * 4 == sb.value
        self.struct = CacheStruct(self.k8.data_ptr(), self.v8t.data_ptr(), self.block.data_ptr(), n_ctx, ld.value,
                                  batch, heads, HEAD_DIM, device.index, 0, 0)
        self.batch, self.heads = batch, heads

    @property
    def ragged(self) -> bool:
        return self.struct.ragged == 1

    def offload(self) -> "OffloadedFP8Cache":
        """A copy of this (filled) cache with K8 / V8^T in page-locked host memory."""
        return OffloadedFP8Cache(self)

    def ctx_len(self) -> list[int]:
        """Per-batch context lengths (n_ctx for every batch unless the fit was ragged)."""
        if not self.ragged:
            return [self.n_ctx] * self.batch
        off = 3 * self.batch * self.heads
        return self.block[off:off + self.batch].view(torch.int32).tolist()

    @property
    def filled(self) -> bool:
        return self.struct.filled == 1

    @property
    def n_ctx(self) -> int:
        return int(self.struct.n_ctx)

    @property
    def ld_v(self) -> int:
        return int(self.struct.ld_v)


# ------------------------------------------------------------- operations

def qscale_fused(q: torch.Tensor, c_h: torch.Tensor, n_len: int, gate: torch.Tensor | None = None,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """LogScale / GatedLogScale of q [B, rows, H, 64] fp16 with shared key length n_len."""
    _want(q, torch.float16, "q", 4)
    B, rows, H, d = q.shape
    _want(c_h, torch.float32, "c_h", 1)
    if gate is not None:
        _want(gate, torch.float16, "gate", 3)
    out = torch.empty_like(q) if out is None else out
    with torch.cuda.device(q.device):
        _check(lib().sdm_qscale_fused(_ptr(q), _ptr(out), B, rows, H, d, int(n_len), _ptr(c_h), _ptr(gate),
                                      _stream(q.device)), "sdm_qscale_fused")
    return out


def fp8_quantize_context(q_scaled: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ctx: int,
                         cache: FP8Cache | None = None, ws: torch.Tensor | None = None):
    """Context-scale e4m3 quantisation.  Returns (q8 [B,H,T,64] uint8, cache)."""
    _want(q_scaled, torch.float16, "q_scaled", 4)
    _want(k, torch.float16, "k", 4)
    _want(v, torch.float16, "v", 4)
    B, T, H, d = q_scaled.shape
    M = T - n_ctx
    dev = q_scaled.device
    cache = FP8Cache(B, n_ctx, H, dev) if cache is None else cache
    q8 = torch.empty((B, H, T, d), dtype=torch.uint8, device=dev)
    need = workspace_size(OP_QUANTIZE_CONTEXT, B, n_ctx, M, H)
    ws = new_workspace(need, dev) if ws is None else ws
    with torch.cuda.device(dev):
        _check(lib().sdm_fp8_quantize_context(_ptr(q_scaled), _ptr(k), _ptr(v), B, n_ctx, M, H, d, _ptr(q8),
                                              ctypes.byref(cache.struct), _ptr(ws), ws.numel(), _stream(dev)),
               "sdm_fp8_quantize_context")
    return q8, cache


def fp8_quantize_context_noalloc(q_scaled: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ctx: int,
                                 cache: FP8Cache | None = None, q8: torch.Tensor | None = None):
    """fp8_quantize_context for callers that cannot provide a workspace: the
    library keeps the amax scratch in a fixed device array of its own (B*H up
    to NOALLOC_MAX_BATCH_HEADS; calls that overlap on the GPU race on it)."""
    _want(q_scaled, torch.float16, "q_scaled", 4)
    _want(k, torch.float16, "k", 4)
    _want(v, torch.float16, "v", 4)
    B, T, H, d = q_scaled.shape
    dev = q_scaled.device
    cache = FP8Cache(B, n_ctx, H, dev) if cache is None else cache
    q8 = torch.empty((B, H, T, d), dtype=torch.uint8, device=dev) if q8 is None else q8
    with torch.cuda.device(dev):
        _check(lib().sdm_fp8_quantize_context_noalloc(_ptr(q_scaled), _ptr(k), _ptr(v), B, n_ctx, T - n_ctx, H, d,
                                                      _ptr(q8), ctypes.byref(cache.struct), _stream(dev)),
               "sdm_fp8_quantize_context_noalloc")
    return q8, cache


def fp8_attention(q8: torch.Tensor, cache: FP8Cache, split: bool = False, out: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None) -> torch.Tensor:
    """Step 3 alone on quantised rows q8 [B,H,rows,64].  Returns out [B,rows,H,64] fp16."""
    _want(q8, torch.uint8, "q8", 4)
    B, H, rows, d = q8.shape
    dev = q8.device
    out = torch.empty((B, rows, H, d), dtype=torch.float16, device=dev) if out is None else out
    need = workspace_size(OP_CACHED_ATTENTION, B, cache.n_ctx, rows, H)
    ws = new_workspace(need, dev) if ws is None else ws
    with torch.cuda.device(dev):
        _check(lib().sdm_fp8_attention(_ptr(q8), B, rows, ctypes.byref(cache.struct), _ptr(out), 1 if split else 0,
                                       _ptr(ws), ws.numel(), _stream(dev)), "sdm_fp8_attention")
    return out


def icl_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ctx: int, c_h: torch.Tensor,
                  gate: torch.Tensor | None = None, cache: FP8Cache | None = None, out: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None, ctx_len=None) -> torch.Tensor:
    """One call of the layer: q [B,T,H,64] raw fp16, k/v [B,N,H,64] fp16 -> out [B,T,H,64] fp16.

    ctx_len (B ints, 1 <= n_b <= n_ctx): ragged batch; rows [n_b, n_ctx) of batch b are padding.
    """
    _want(q, torch.float16, "q", 4)
    _want(k, torch.float16, "k", 4)
    _want(v, torch.float16, "v", 4)
    _want(c_h, torch.float32, "c_h", 1)
    if gate is not None:
        _want(gate, torch.float16, "gate", 3)
    B, T, H, d = q.shape
    M = T - n_ctx
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    need = workspace_size(OP_ICL_ATTENTION, B, n_ctx, M, H, keep_cache=cache is not None)
    ws = new_workspace(need, dev) if ws is None else ws
    cs = None if cache is None else ctypes.byref(cache.struct)
    with torch.cuda.device(dev):
        if ctx_len is None:
            _check(lib().sdm_icl_attention(_ptr(q), _ptr(k), _ptr(v), B, n_ctx, M, H, d, _ptr(c_h), _ptr(gate),
                                           _ptr(out), cs, _ptr(ws), ws.numel(), _stream(dev)), "sdm_icl_attention")
        else:
            _check(lib().sdm_icl_attention_ragged(_ptr(q), _ptr(k), _ptr(v), B, n_ctx, M, H, d,
                                                  _ctx_len_array(ctx_len, B), _ptr(c_h), _ptr(gate), _ptr(out), cs,
                                                  _ptr(ws), ws.numel(), _stream(dev)), "sdm_icl_attention_ragged")
    return out


def cached_attention(q: torch.Tensor, cache: FP8Cache, c_h: torch.Tensor, gate: torch.Tensor | None = None,
                     out: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Cached prediction: q [B,M,H,64] raw fp16 against a filled cache -> out [B,M,H,64] fp16."""
    _want(q, torch.float16, "q", 4)
    _want(c_h, torch.float32, "c_h", 1)
    if gate is not None:
        _want(gate, torch.float16, "gate", 3)
    B, M, H, d = q.shape
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    need = workspace_size(OP_CACHED_ATTENTION, B, cache.n_ctx, M, H)
    ws = new_workspace(need, dev) if ws is None else ws
    with torch.cuda.device(dev):
        _check(lib().sdm_cached_attention(_ptr(q), B, M, H, d, ctypes.byref(cache.struct), _ptr(c_h), _ptr(gate),
                                          _ptr(out), _ptr(ws), ws.numel(), _stream(dev)), "sdm_cached_attention")
    return out


def fp8_eligible(n_unmasked_ctx: int, final_layer: bool = False) -> bool:
    """The precision rule: FP8 attention only on a non-final ICL layer above 8,192 unmasked context rows."""
    return bool(lib().sdm_fp8_eligible(int(n_unmasked_ctx), 1 if final_layer else 0))


def icl_attention_f16(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ctx: int, c_h: torch.Tensor | None,
                      gate: torch.Tensor | None = None, out: torch.Tensor | None = None,
                      ws: torch.Tensor | None = None, ctx_len=None) -> torch.Tensor:
    """Normal-precision layer call: q [B,T,H,64] raw fp16, k/v [B,N,H,64] fp16 -> out [B,T,H,64] fp16.

    c_h None: no query scaling (q is used as given; gate must be None).  ctx_len: ragged batch
    as for icl_attention.
    """
    _want(q, torch.float16, "q", 4)
    _want(k, torch.float16, "k", 4)
    _want(v, torch.float16, "v", 4)
    if c_h is not None:
        _want(c_h, torch.float32, "c_h", 1)
    if gate is not None:
        _want(gate, torch.float16, "gate", 3)
    B, T, H, d = q.shape
    M = T - n_ctx
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    need = workspace_size(OP_ICL_ATTENTION_F16, B, n_ctx, M, H)
    ws = new_workspace(need, dev) if ws is None else ws
    with torch.cuda.device(dev):
        if ctx_len is None:
            _check(lib().sdm_icl_attention_f16(_ptr(q), _ptr(k), _ptr(v), B, n_ctx, M, H, d, _ptr(c_h),
                                               _ptr(gate), _ptr(out), _ptr(ws), ws.numel(), _stream(dev)),
                   "sdm_icl_attention_f16")
        else:
            _check(lib().sdm_icl_attention_f16_ragged(_ptr(q), _ptr(k), _ptr(v), B, n_ctx, M, H, d,
                                                      _ctx_len_array(ctx_len, B), _ptr(c_h), _ptr(gate), _ptr(out),
                                                      _ptr(ws), ws.numel(), _stream(dev)),
                   "sdm_icl_attention_f16_ragged")
    return out


def icl_layer(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ctx: int, c_h: torch.Tensor,
              gate: torch.Tensor | None = None, final_layer: bool = False, cache: FP8Cache | None = None,
              out: torch.Tensor | None = None, ctx_len=None) -> torch.Tensor:
    """One ICL attention layer with the precision rule applied: FP8 (icl_attention) when
    fp8_eligible(n, final_layer), else normal precision (icl_attention_f16).  n is the number of
    unmasked context rows: n_ctx, or for a ragged batch the smallest n_b (FP8 only when every
    estimator of the batch qualifies).  A cache can only be filled on the FP8 path."""
    n_unmasked = n_ctx if ctx_len is None else min(int(x) for x in ctx_len)
    if fp8_eligible(n_unmasked, final_layer):
        return icl_attention(q, k, v, n_ctx, c_h, gate=gate, cache=cache, out=out, ctx_len=ctx_len)
    if cache is not None:
        raise ValueError("an FP8 cache is filled only by an FP8-eligible layer "
                         f"(unmasked context rows={n_unmasked}, final_layer={final_layer})")
    return icl_attention_f16(q, k, v, n_ctx, c_h, gate=gate, out=out, ctx_len=ctx_len)


class OffloadedFP8Cache:
    """An FP8 cache whose K8 / V8^T live in page-locked host memory; the scales block (a few
    KB) stays on the device.  Read by cached_attention_offload one split-KV chunk at a time."""

    def __init__(self, cache: FP8Cache):
        if not cache.filled:
            raise ValueError("only a filled cache can be offloaded")
        torch.cuda.current_stream(cache.k8.device).synchronize()
        self.k8 = torch.empty(cache.k8.shape, dtype=torch.uint8, pin_memory=True)
        self.v8t = torch.empty(cache.v8t.shape, dtype=torch.uint8, pin_memory=True)
        self.k8.copy_(cache.k8)
        self.v8t.copy_(cache.v8t)
        self.block = cache.block.clone()
        c = cache.struct
        self.struct = CacheStruct(self.k8.data_ptr(), self.v8t.data_ptr(), self.block.data_ptr(), c.n_ctx, c.ld_v,
                                  c.batch, c.heads, c.head_dim, c.device, c.filled, c.ragged)
        self.device = cache.k8.device
        self.n_ctx = int(c.n_ctx)


_copy_streams: dict = {}


def cached_attention_offload(q: torch.Tensor, cache: OffloadedFP8Cache, c_h: torch.Tensor,
                             gate: torch.Tensor | None = None, out: torch.Tensor | None = None,
                             ws: torch.Tensor | None = None, copy_stream=None) -> torch.Tensor:
    """Cached prediction against an offloaded cache: q [B,M,H,64] raw fp16 -> out [B,M,H,64] fp16,
    identical to cached_attention on the same cache.  Host-to-device copies run on copy_stream
    (default: one side stream per device), overlapped with the attention."""
    _want(q, torch.float16, "q", 4)
    _want(c_h, torch.float32, "c_h", 1)
    if gate is not None:
        _want(gate, torch.float16, "gate", 3)
    B, M, H, d = q.shape
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    need = workspace_size(OP_CACHED_ATTENTION_OFFLOAD, B, cache.n_ctx, M, H)
    ws = new_workspace(need, dev) if ws is None else ws
    if copy_stream is None:
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        if key not in _copy_streams:
            _copy_streams[key] = torch.cuda.Stream(device=dev)
        copy_stream = _copy_streams[key]
    with torch.cuda.device(dev):
        _check(lib().sdm_cached_attention_offload(_ptr(q), B, M, H, d, ctypes.byref(cache.struct), _ptr(c_h),
                                                  _ptr(gate), _ptr(out), _ptr(ws), ws.numel(), _stream(dev),
                                                  ctypes.c_void_p(copy_stream.cuda_stream)),
               "sdm_cached_attention_offload")
    return out


def gqa_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, qo_indptr, kv_indptr, causal: bool = True,
                out: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Ragged grouped-query prefill: q [total_q, Hq, 128], k / v [total_kv, Hkv, 128] bf16, host indptr
    sequences of batch + 1 offsets -> out [total_q, Hq, 128] bf16."""
    _want(q, torch.bfloat16, "q", 3)
    _want(k, torch.bfloat16, "k", 3)
    _want(v, torch.bfloat16, "v", 3)
    qo = (ctypes.c_int64 * len(qo_indptr))(*[int(x) for x in qo_indptr])
    kvo = (ctypes.c_int64 * len(kv_indptr))(*[int(x) for x in kv_indptr])
    if len(qo_indptr) != len(kv_indptr):
        raise ValueError("qo_indptr and kv_indptr must have the same length")
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    if ws is None:
        ws = new_workspace(gqa_prefill_workspace_size(qo_indptr, kv_indptr, q.shape[1], k.shape[1], causal), dev)
    with torch.cuda.device(dev):
        _check(lib().sdm_gqa_prefill(_ptr(q), _ptr(k), _ptr(v), qo, kvo, len(qo_indptr) - 1, q.shape[1], k.shape[1],
                                     q.shape[2], 1 if causal else 0, _ptr(out), _ptr(ws), ws.numel(), _stream(dev)),
               "sdm_gqa_prefill")
    return out


def gqa_prefill_workspace_size(qo_indptr, kv_indptr, q_heads: int, kv_heads: int, causal: bool = True) -> int:
    """Workspace bytes sdm_gqa_prefill needs for this batch (0 for an invalid batch)."""
    qo = (ctypes.c_int64 * len(qo_indptr))(*[int(x) for x in qo_indptr])
    kvo = (ctypes.c_int64 * len(kv_indptr))(*[int(x) for x in kv_indptr])
    return int(lib().sdm_gqa_prefill_workspace_size(qo, kvo, len(qo_indptr) - 1, q_heads, kv_heads, 128,
                                                    1 if causal else 0))


# ------------------------------------------------------ sharded quantisation

def context_amax(q: torch.Tensor, k: torch.Tensor | None, v: torch.Tensor | None, n_ctx: int, n_len: int,
                 c_h: torch.Tensor | None = None, gate: torch.Tensor | None = None,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """[3, B, H] fp32 maxima of |Q'|, |K|, |V| over context rows [0, n_ctx) of a slice
    (sdm_context_amax).  q [B, q_rows, H, 64] is raw (query scaling with n_len, c_h,
    gate fused) or, with c_h None, already scaled."""
    _want(q, torch.float16, "q", 4)
    B, q_rows, H, d = q.shape
    if n_ctx > 0:
        _want(k, torch.float16, "k", 4)
        _want(v, torch.float16, "v", 4)
    if c_h is not None:
        _want(c_h, torch.float32, "c_h", 1)
    if gate is not None:
        _want(gate, torch.float16, "gate", 3)
    dev = q.device
    out = torch.empty((3, B, H), dtype=torch.float32, device=dev) if out is None else out
    with torch.cuda.device(dev):
        _check(lib().sdm_context_amax(_ptr(q), _ptr(k if n_ctx > 0 else None), _ptr(v if n_ctx > 0 else None), B,
                                      int(n_ctx), q_rows, H, d, int(n_len), _ptr(c_h), _ptr(gate), _ptr(out),
                                      _stream(dev)), "sdm_context_amax")
    return out


def quantize_with_scales(q: torch.Tensor, k: torch.Tensor | None, v: torch.Tensor | None, n_ctx: int, n_len: int,
                         amax: torch.Tensor, c_h: torch.Tensor | None = None, gate: torch.Tensor | None = None,
                         ld_k: int | None = None, ld_v: int | None = None, scales: torch.Tensor | None = None):
    """Scales amax/448 and the e4m3 codes of a slice's rows (sdm_quantize_with_scales).
    q [B, n_ctx + n_query, H, 64]; k, v [B, n_ctx, H, 64].  Returns (q8 [B,H,T,64],
    k8 [B,H,ld_k,64] (rows [0, n_ctx) written), v8t [B,H,64,ld_v], scales [3,B,H])."""
    _want(q, torch.float16, "q", 4)
    _want(amax, torch.float32, "amax", 3)
    B, T, H, d = q.shape
    dev = q.device
    ld_k = n_ctx if ld_k is None else int(ld_k)
    ld_v = max(KV_TILE, -(-n_ctx // KV_TILE) * KV_TILE) if ld_v is None else int(ld_v)
    q8 = torch.empty((B, H, T, d), dtype=torch.uint8, device=dev)
    k8 = torch.empty((B, H, ld_k, d), dtype=torch.uint8, device=dev)
    v8t = torch.empty((B, H, d, ld_v), dtype=torch.uint8, device=dev)
    scales = torch.empty((3, B, H), dtype=torch.float32, device=dev) if scales is None else scales
    if n_ctx > 0:
        _want(k, torch.float16, "k", 4)
        _want(v, torch.float16, "v", 4)
    with torch.cuda.device(dev):
        _check(lib().sdm_quantize_with_scales(_ptr(q), _ptr(k if n_ctx > 0 else None), _ptr(v if n_ctx > 0 else None),
                                              B, int(n_ctx), T - int(n_ctx), H, d, int(n_len), _ptr(c_h), _ptr(gate),
                                              _ptr(amax), _ptr(scales), _ptr(q8),
                                              _ptr(k8 if n_ctx > 0 else None), ld_k,
                                              _ptr(v8t if n_ctx > 0 else None), ld_v, _stream(dev)),
               "sdm_quantize_with_scales")
    return q8, k8, v8t, scales


def cache_put_rows(cache: FP8Cache, k8_rows: torch.Tensor, v8t_cols: torch.Tensor, row0: int, n: int) -> None:
    """Place rows [0, n) of a slice's K8 planes [B,H,ld_k,64] and columns [0, n) of its
    V8^T rows [B,H,64,ld_v] at global context row row0 of the cache (sdm_cache_put_rows)."""
    _want(k8_rows, torch.uint8, "k8_rows", 4)
    _want(v8t_cols, torch.uint8, "v8t_cols", 4)
    dev = k8_rows.device
    with torch.cuda.device(dev):
        _check(lib().sdm_cache_put_rows(ctypes.byref(cache.struct), _ptr(k8_rows), k8_rows.shape[2], _ptr(v8t_cols),
                                        v8t_cols.shape[3], int(row0), int(n), _stream(dev)), "sdm_cache_put_rows")


# ------------------------------------------------- cached prediction by chunks

def split_count(n_ctx: int) -> int:
    """Number of split-KV chunks of cached prediction for an n_ctx-key context."""
    return -(-int(n_ctx) // split_keys(n_ctx))


def partial_buffers(cache: FP8Cache, n_query: int, chunks: int | None = None):
    """Zeroed split-KV partial buffers (acc [S,B,H,M,64], (m2, l) [S,B,H,M,2]) for `chunks`
    chunks (default: all of the cache's)."""
    S = split_count(cache.n_ctx) if chunks is None else int(chunks)
    dev = cache.k8.device
    return (torch.zeros((S, cache.batch, cache.heads, n_query, HEAD_DIM), dtype=torch.float32, device=dev),
            torch.zeros((S, cache.batch, cache.heads, n_query, 2), dtype=torch.float32, device=dev))


def cached_partials(q: torch.Tensor, cache: FP8Cache, k8_slice: torch.Tensor, v8t_slice: torch.Tensor, c0: int,
                    c1: int, c_h: torch.Tensor, part_acc: torch.Tensor, part_ml: torch.Tensor,
                    gate: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> None:
    """Partials of chunks [c0, c1) from the keys of those chunks only (sdm_cached_partials):
    k8_slice [B,H,n,64], v8t_slice [B,H,64,ld]; writes part_acc / part_ml rows c0..c1-1."""
    _want(q, torch.float16, "q", 4)
    _want(k8_slice, torch.uint8, "k8_slice", 4)
    _want(v8t_slice, torch.uint8, "v8t_slice", 4)
    B, M, H, d = q.shape
    dev = q.device
    ws = new_workspace(workspace_size(OP_CACHED_PARTIALS, B, cache.n_ctx, M, H), dev) if ws is None else ws
    with torch.cuda.device(dev):
        _check(lib().sdm_cached_partials(_ptr(q), B, M, H, d, ctypes.byref(cache.struct), _ptr(k8_slice),
                                         _ptr(v8t_slice), v8t_slice.shape[3], int(c0), int(c1), _ptr(c_h),
                                         _ptr(gate), _ptr(part_acc), _ptr(part_ml), _ptr(ws), ws.numel(),
                                         _stream(dev)), "sdm_cached_partials")


def cached_combine(part_acc: torch.Tensor, part_ml: torch.Tensor, cache: FP8Cache, n_query: int,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """The fixed-order combine of all chunks' partials (sdm_cached_combine): out [B,M,H,64] fp16."""
    dev = part_acc.device
    out = torch.empty((cache.batch, n_query, cache.heads, HEAD_DIM), dtype=torch.float16, device=dev) \
        if out is None else out
    with torch.cuda.device(dev):
        _check(lib().sdm_cached_combine(_ptr(part_acc), _ptr(part_ml), cache.batch, int(n_query), cache.heads,
                                        HEAD_DIM, ctypes.byref(cache.struct), _ptr(out), _stream(dev)),
               "sdm_cached_combine")
    return out
