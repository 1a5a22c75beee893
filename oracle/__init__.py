"""CPU oracle for the FP8 in-context-learning attention layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the library under
``fp8_quant_logscale_b200`` never does.  It shares no code with the CUDA path.

The arithmetic lives in ``oracle.c`` (plain C, OpenMP over rows, built with
``-O2 -ffp-contract=off`` and no fast-math).  This module only compiles it and
marshals numpy arrays through ctypes.  Every function is pinned by the
``-m "not gpu"`` tests against library casts, closed forms, brute force and
invariants; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# KV tile (online-softmax block) and cached-prediction split length that the
# layer is defined with.  These are algorithm parameters, restated here on the
# oracle side from the layer's specification: 128-key tiles; the cached path
# cuts the keys into chunks whose length depends on N only -- about 32 chunks,
# each a multiple of 128 keys, clamped to [1024, 16384].
KV_TILE = 128


# Ambiguity radius of a key's e4m3 probability code for an implementation that
# forms the probabilities in single precision (attention()'s delta and kappa):
#  - delta: the 2^x evaluation (an FMA-pipe polynomial erring by at most 2.71e-6
#    relative, MUFU ex2.approx by 2^-22) with a margin;
#  - kappa per base-2 unit of |m2| + |t_j|: the logit passes through fp32 numbers of
#    that size -- z accumulated from 64 exact products in fp32 on a tensor core,
#    the scale c2 (three roundings), the shifted maximum m2 and the shift t (one
#    each) -- and a relative error e of the logit is ln2 * e in the probability;
#    32 roundings (2^-24 each) of that size cover them with a margin of about 2.
# Where the definition's probability lies within that distance of a rounding
# midpoint, either neighbouring code is what a correct fp32 implementation may
# produce; attention()'s allowance bounds the output change of any such choice.
FP32_AMBIGUITY = dict(delta=4e-6, kappa=32 * 2.0 ** -24 * float(np.log(2.0)))


def split_keys(n_ctx: int) -> int:
    """Chunk length of the cached-prediction split for an n_ctx-key context."""
    per = -(-n_ctx // (32 * KV_TILE)) * KV_TILE
    return min(16384, max(1024, per))


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double


def _declare(L):
    L.orc_f16_decode.restype = _D
    L.orc_f16_decode.argtypes = [ctypes.c_uint16]
    L.orc_f16_encode.restype = ctypes.c_uint16
    L.orc_f16_encode.argtypes = [_D]
    L.orc_e4m3_decode.restype = _D
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [_D]
    for name in ("orc_f16_encode_array", "orc_f16_decode_array",
                 "orc_e4m3_encode_array", "orc_e4m3_decode_array"):
        getattr(L, name).restype = None
        getattr(L, name).argtypes = [_P, _I64, _P]
    L.orc_log_length.restype = ctypes.c_float
    L.orc_log_length.argtypes = [_I64]
    L.orc_qscale.restype = None
    L.orc_qscale.argtypes = [_P, _I, _I64, _I, _I, _I64, _P, _P, _P]
    L.orc_context_scales.restype = None
    L.orc_context_scales.argtypes = [_P, _I, _I64, _I64, _I, _I, _P]
    L.orc_quantize.restype = None
    L.orc_quantize.argtypes = [_P, _I, _I64, _I, _I, _P, _P]
    L.orc_attention.restype = None
    L.orc_attention.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I64, _I64, _I,
                                _P, _I64, _I64, _I64, _I, _I, _D, _D, _P, _P, _P]
    L.orc_attention_partials.restype = None
    L.orc_attention_partials.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I64, _I64, _I64, _I, _P, _I64, _I64, _I64,
                                         _I64, _P, _P, _P]
    L.orc_attention_exact.restype = None
    L.orc_attention_exact.argtypes = [_P, _P, _P, _I, _I, _I64, _I64, _I, _P, _I64, _P]
    L.orc_num_threads.restype = _I
    L.orc_num_threads.argtypes = []
    L.orc_set_num_threads.restype = None
    L.orc_set_num_threads.argtypes = [_I]


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _bits16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    return x.view(np.uint16) if x.dtype == np.float16 else x.astype(np.uint16)


# --- codecs -----------------------------------------------------------------

def f16_encode(y) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, np.uint16)
    lib().orc_f16_encode_array(_ptr(y), y.size, _ptr(out))
    return out


def f16_decode(h) -> np.ndarray:
    h = _bits16(h)
    out = np.empty(h.shape, np.float64)
    lib().orc_f16_decode_array(_ptr(h), h.size, _ptr(out))
    return out


def e4m3_encode(y) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, np.uint8)
    lib().orc_e4m3_encode_array(_ptr(y), y.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def log_length(n: int) -> float:
    return float(lib().orc_log_length(int(n)))


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the following oracle calls (OpenMP)."""
    lib().orc_set_num_threads(int(n))


# --- the layer ----------------------------------------------------------------

def qscale(q: np.ndarray, n: int, c_h: np.ndarray, gate: np.ndarray | None = None) -> np.ndarray:
    """LogScale (gate None) or GatedLogScale of q [B, rows, H, d] fp16 -> fp16."""
    B, rows, H, d = q.shape
    qb = _bits16(q)
    c = np.ascontiguousarray(c_h, dtype=np.float32)
    gb = None if gate is None else _bits16(gate)
    if gb is not None:
        assert gb.shape == (B, rows, H)
    out = np.empty(q.shape, np.uint16)
    lib().orc_qscale(_ptr(qb), B, rows, H, d, int(n), _ptr(c), _ptr(gb), _ptr(out))
    return out.view(np.float16)


def context_scales(x: np.ndarray, n_ctx: int) -> np.ndarray:
    """Per-(b, h) scale amax/448 over the first n_ctx rows of x [B, rows, H, d]."""
    B, rows, H, d = x.shape
    xb = _bits16(x)
    out = np.empty((B, H), np.float32)
    lib().orc_context_scales(_ptr(xb), B, rows, int(n_ctx), H, d, _ptr(out))
    return out


def quantize(x: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """e4m3 codes [B, H, rows, d] of x [B, rows, H, d] / scale[b, h]."""
    B, rows, H, d = x.shape
    xb = _bits16(x)
    s = np.ascontiguousarray(scale, dtype=np.float32).reshape(B, H)
    out = np.empty((B, H, rows, d), np.uint8)
    lib().orc_quantize(_ptr(xb), B, rows, H, d, _ptr(s), _ptr(out))
    return out


ARITH = {"definition": 0, "fp32": 1}


def attention(q8, k8, v8, s_q, s_k, s_v, rows=None, bc: int = KV_TILE, split: int = 0,
              quant_p: bool = True, delta: float = 0.0, kappa: float = 0.0, arith: str = "definition"):
    """FP8 online-softmax attention of the selected rows of q8 to all keys.

    q8 [B,H,T,d], k8/v8 [B,H,N,d] uint8 codes; s_* [B,H] fp32.
    arith: "definition" (the oracle: logits, exp and sums in double) or "fp32"
    (a diagnostic: the single-precision sequence a tensor-core kernel takes).
    delta, kappa: the ambiguity radius delta + kappa * (|m2| + |t_j|) of key j
    (base-2 units); the returned allowance bounds the output change when any set
    of keys within that relative distance of an e4m3 midpoint takes its other code.
    Returns (out16 [B,n,H,d] fp16, out [B,n,H,d] f64, allowance [B,n,H,d] f64).
    """
    q8 = np.ascontiguousarray(q8, np.uint8)
    k8 = np.ascontiguousarray(k8, np.uint8)
    v8 = np.ascontiguousarray(v8, np.uint8)
    B, H, T, d = q8.shape
    N = k8.shape[2]
    assert k8.shape == (B, H, N, d) and v8.shape == (B, H, N, d)
    if rows is None:
        rows = np.arange(T, dtype=np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    n = rows.size
    sq = np.ascontiguousarray(s_q, np.float32).reshape(B * H)
    sk = np.ascontiguousarray(s_k, np.float32).reshape(B * H)
    sv = np.ascontiguousarray(s_v, np.float32).reshape(B * H)
    out16 = np.empty((B, n, H, d), np.uint16)
    out = np.empty((B, n, H, d), np.float64)
    allow = np.empty((B, n, H, d), np.float64)
    lib().orc_attention(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv),
                        B, H, T, N, d, _ptr(rows), n, int(bc), int(split),
                        1 if quant_p else 0, ARITH[arith], float(delta), float(kappa),
                        _ptr(out16), _ptr(out), _ptr(allow))
    return out16.view(np.float16), out, allow


def attention_partials(q8, k8_slice, v8_slice, s_q, s_k, n_ctx: int, split: int, c0: int, c1: int, rows=None):
    """Per-chunk partial states (definition arithmetic) of chunks [c0, c1) of `split` keys,
    from the keys of those chunks only: k8_slice / v8_slice [B,H,n_slice,d] hold keys
    [c0 split, c0 split + n_slice) of the n_ctx.  Returns m [C,B,H,n] (natural-log units),
    l [C,B,H,n] and acc [C,B,H,n,d]; combine_partials of all chunks is attention(split=split)."""
    q8 = np.ascontiguousarray(q8, np.uint8)
    k8s = np.ascontiguousarray(k8_slice, np.uint8)
    v8s = np.ascontiguousarray(v8_slice, np.uint8)
    B, H, T, d = q8.shape
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    C, n = c1 - c0, rows.size
    m = np.empty((C, B, H, n))
    l = np.empty((C, B, H, n))
    acc = np.empty((C, B, H, n, d))
    sq = np.ascontiguousarray(s_q, np.float32).reshape(B * H)
    sk = np.ascontiguousarray(s_k, np.float32).reshape(B * H)
    lib().orc_attention_partials(_ptr(q8), _ptr(k8s), _ptr(v8s), _ptr(sq), _ptr(sk), B, H, T, int(n_ctx),
                                 k8s.shape[2], d, _ptr(rows), n, int(split), int(c0), int(c1),
                                 _ptr(m), _ptr(l), _ptr(acc))
    return m, l, acc


def combine_partials(m, l, acc, s_v):
    """The fixed-order combine of every chunk's state: M = max_s m_s, w_s = exp(m_s - M),
    O = (sum_s w_s acc_s) s_v / (sum_s w_s l_s).  m, l [S,B,H,n], acc [S,B,H,n,d], s_v [B,H].
    Returns O [B,n,H,d] (double)."""
    M = m.max(axis=0)
    w = np.where(np.isneginf(m), 0.0, np.exp(m - M))
    L = (w * l).sum(axis=0)
    ACC = (w[..., None] * acc).sum(axis=0)
    o = ACC * np.asarray(s_v, np.float64)[..., None, None] / L[..., None]
    return o.transpose(0, 2, 1, 3)


def attention_exact(q, k, v, rows=None):
    """Double-precision softmax(q k^T / sqrt(d)) v, no quantisation.

    q [B,T,H,d], k/v [B,N,H,d] fp16.  Returns [B,n,H,d] f64.
    """
    B, T, H, d = q.shape
    N = k.shape[1]
    if rows is None:
        rows = np.arange(T, dtype=np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.empty((B, rows.size, H, d), np.float64)
    # keep the (possibly copied) contiguous inputs alive for the duration of the call
    qb, kb, vb = _bits16(q), _bits16(k), _bits16(v)
    lib().orc_attention_exact(_ptr(qb), _ptr(kb), _ptr(vb), B, H, T, N, d, _ptr(rows), rows.size, _ptr(out))
    return out


def layer(q, k, v, n_ctx: int, c_h, gate=None, rows=None, split: int = 0, delta: float = 0.0,
          kappa: float = 0.0):
    """All steps of the layer on the CPU: qscale -> scales -> e4m3 -> attention.

    q [B,T,H,d] fp16 (T = n_ctx + queries), k/v [B,n_ctx,H,d] fp16.
    Returns a dict with every intermediate (for staged parity checks).
    """
    qs = qscale(q, n_ctx, c_h, gate)
    s_q = context_scales(qs, n_ctx)
    s_k = context_scales(k, n_ctx)
    s_v = context_scales(v, n_ctx)
    q8 = quantize(qs, s_q)
    k8 = quantize(k, s_k)
    v8 = quantize(v, s_v)
    o16, o, allow = attention(q8, k8, v8, s_q, s_k, s_v, rows=rows, split=split, delta=delta, kappa=kappa)
    return dict(q_scaled=qs, s_q=s_q, s_k=s_k, s_v=s_v, q8=q8, k8=k8, v8=v8,
                out16=o16, out=o, allow=allow)


# --- ragged batches (batched estimators with padded contexts) ------------------

def _ragged_rows(n_b: int, N: int, T: int) -> np.ndarray:
    """Rows of a padded batch that the layer computes: context [0, n_b) and queries [N, T)."""
    return np.concatenate([np.arange(n_b), np.arange(N, T)]).astype(np.int64)


def layer_ragged(q, k, v, ctx_len, c_h, gate=None, split: int = 0, delta: float = 0.0, kappa: float = 0.0):
    """A batch of estimators whose contexts are padded to N rows ("unmasked context
    rows", [FP8 3/4] opening section): batch b is `layer` on its own rows only --
    query scaling with n = n_b, scales from rows [0, n_b), context rows [0, n_b)
    and query rows [N, T) attending to keys [0, n_b).  Padding rows [n_b, N) take
    part in nothing; their outputs and e4m3 codes are zero.

    q [B,T,H,d], k/v [B,N,H,d] fp16, ctx_len [B] with 1 <= n_b <= N.
    Returns out16/out/allow [B,T,H,d], s_q/s_k/s_v [B,H], q8 [B,H,T,d], k8/v8 [B,H,N,d]
    and q_scaled [B,T,H,d] (padding rows zero).
    """
    B, T, H, d = q.shape
    N = k.shape[1]
    ctx_len = [int(x) for x in ctx_len]
    assert len(ctx_len) == B and all(1 <= n <= N for n in ctx_len)
    res = dict(out16=np.zeros((B, T, H, d), np.float16), out=np.zeros((B, T, H, d)),
               allow=np.zeros((B, T, H, d)), s_q=np.empty((B, H), np.float32), s_k=np.empty((B, H), np.float32),
               s_v=np.empty((B, H), np.float32), q8=np.zeros((B, H, T, d), np.uint8),
               k8=np.zeros((B, H, N, d), np.uint8), v8=np.zeros((B, H, N, d), np.uint8),
               q_scaled=np.zeros((B, T, H, d), np.float16))
    for b, n in enumerate(ctx_len):
        rows = _ragged_rows(n, N, T)
        g = None if gate is None else np.ascontiguousarray(gate[b:b + 1, rows])
        r = layer(np.ascontiguousarray(q[b:b + 1, rows]), np.ascontiguousarray(k[b:b + 1, :n]),
                  np.ascontiguousarray(v[b:b + 1, :n]), n, c_h, g, split=split, delta=delta, kappa=kappa)
        for key in ("out16", "out", "allow", "q_scaled"):
            res[key][b, rows] = r[key][0]
        for key in ("s_q", "s_k", "s_v"):
            res[key][b] = r[key][0]
        res["q8"][b][:, rows] = r["q8"][0]
        res["k8"][b][:, :n] = r["k8"][0]
        res["v8"][b][:, :n] = r["v8"][0]
    return res


def attention_exact_ragged(q, k, v, ctx_len, rows=None):
    """Double-precision attention of a padded batch: row i of batch b attends to keys
    [0, n_b); rows [n_b, N) are padding (0).  q [B,T,H,d] (already query-scaled), k/v
    [B,N,H,d].  Returns [B,n,H,d] f64 for the selected rows (all rows if None)."""
    B, T, H, d = q.shape
    N = k.shape[1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    out = np.zeros((B, rows.size, H, d))
    for b, n in enumerate(int(x) for x in ctx_len):
        sel = np.nonzero((rows < n) | (rows >= N))[0]
        if sel.size:
            out[b, sel] = attention_exact(np.ascontiguousarray(q[b:b + 1]), np.ascontiguousarray(k[b:b + 1, :n]),
                                          np.ascontiguousarray(v[b:b + 1, :n]), rows=rows[sel])[0]
    return out


# --- ragged grouped-query prefill (bf16 in, exact softmax) ----------------------

def bf16_decode(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 (a bf16 value is the top 16 bits of a float32)."""
    b = np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def gqa_prefill(q, k, v, qo_indptr, kv_indptr, q_heads: int, kv_heads: int, causal: bool = True):
    """Attention of a packed ragged batch with grouped-query heads, in double precision.

    Sequence b owns query tokens [qo[b], qo[b+1]) and key/value tokens [kv[b], kv[b+1]);
    query head h reads key/value head h // (q_heads / kv_heads); scores are scaled by
    1/sqrt(d).  Causal (the queries are the last q_len of the kv_len tokens): query i
    attends keys j <= kv_len - q_len + i.  q [Tq, Hq, d], k/v [Tkv, Hkv, d] as bf16 bits.
    Returns out [Tq, Hq, d] float64.
    """
    qd, kd, vd = bf16_decode(q), bf16_decode(k), bf16_decode(v)
    Tq, Hq, d = qd.shape
    assert Hq == q_heads and kd.shape[1] == kv_heads and q_heads % kv_heads == 0
    G = q_heads // kv_heads
    out = np.zeros((Tq, Hq, d))
    for b in range(len(qo_indptr) - 1):
        q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        k0, k1 = int(kv_indptr[b]), int(kv_indptr[b + 1])
        nq, nk = q1 - q0, k1 - k0
        if nq == 0:
            continue
        allowed = np.ones((nq, nk), bool)
        if causal:
            assert nk >= nq, "causal prefill needs kv_len >= q_len"
            allowed = np.arange(nk)[None, :] <= (nk - nq + np.arange(nq))[:, None]
        for h in range(Hq):
            g = h // G
            s = (qd[q0:q1, h] @ kd[k0:k1, g].T) / np.sqrt(d)
            s = np.where(allowed, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            out[q0:q1, h] = (p / p.sum(axis=1, keepdims=True)) @ vd[k0:k1, g]
    return out
