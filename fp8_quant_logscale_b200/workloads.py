"""Seeded synthetic inputs for the FP8 ICL-attention layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it.  The pages measure on TabArena / OpenML datasets with pretrained
TabICLv2 and Kumo checkpoints ("[FP8 3/4] Integrate FP8 attention and caching
into TabICLv2", timing table: 16,384 to 524,288 context rows, 1,024 query
rows); none of that is available, so these seeded tensors of the same shapes
stand in for the attention layer's Q/K/V.

Generation recipe: numpy ``Generator(PCG64)``
streams keyed by (seed, tensor id, chunk index) over 2^22-element chunks,
standard normal in float32, rounded to fp16 (RNE); per-(tensor, head) factors
and the 0.1% x20 outliers, where a workload asks for them, come from their own
streams.  c_h ~ U(0.5, 1.5) fp32 per head; gate g ~ N(0, 1) fp16 per (row, head).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK = 1 << 22
_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "gate": 4, "c_h": 5, "head_factor": 6, "outlier": 7, "queries": 8,
               "ctx_len": 9}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_ctx: int            # N context rows
    n_query: int          # M query rows
    heads: int            # H
    head_dim: int = 64
    batch: int = 1
    gated: bool = False   # GatedLogScale with g ~ N(0, 1)
    head_factor: tuple | None = None   # per-(tensor, head) U(lo, hi) multiplier
    outliers: float = 0.0  # fraction of elements multiplied by outlier_scale
    outlier_scale: float = 20.0
    cached: bool = False   # cached prediction against an n_ctx-row cache
    ragged: tuple | None = None  # batch b has n_b ~ U{floor(lo*N)+1 .. floor(hi*N)} unmasked context rows
    seed: int = 0
    description: str = ""

    @property
    def rows(self) -> int:
        return self.n_ctx + self.n_query


# The five workloads of the layer's specification, named by what they are.
WORKLOADS = {
    "icl_n1k_m128_h4": Workload(
        "icl_n1k_m128_h4", 1024, 128, 4, seed=1,
        description="N=1024 context rows, M=128 queries, H=4, d=64, fp16 N(0,1); LogScale n=1024; "
                    "context self-attention + query->context cross-attention"),
    "icl_n16k_m1k_h8": Workload(
        "icl_n16k_m1k_h8", 16384, 1024, 8, head_factor=(0.5, 4.0), seed=2,
        description="N=16384, M=1024, H=8, d=64, fp16 N(0,1) scaled per (tensor, head) by U(0.5,4); LogScale"),
    "icl_n128k_m1k_h8_gated": Workload(
        "icl_n128k_m1k_h8_gated", 131072, 1024, 8, gated=True, outliers=0.001, seed=3,
        description="N=131072, M=1024, H=8, d=64, fp16 N(0,1) with 0.1% outliers x20; GatedLogScale g~N(0,1)"),
    "icl_n512k_m1k_h8": Workload(
        "icl_n512k_m1k_h8", 524288, 1024, 8, seed=4,
        description="N=524288, M=1024, H=8, d=64, fp16 N(0,1); LogScale; FP8 self + cross attention"),
    "icl_n256k_m1k_h8": Workload(
        "icl_n256k_m1k_h8", 262144, 1024, 8, seed=9,
        description="N=262144, M=1024, H=8, d=64, fp16 N(0,1); LogScale: the 512K workload's recipe at half "
                    "the context, small enough for a full ncu capture of the long-context attention"),
    "icl_n128k_m1k_h8_flat": Workload(
        "icl_n128k_m1k_h8_flat", 131072, 1024, 8, head_factor=(0.01, 0.02), seed=8,
        description="N=131072, M=1024, H=8, d=64, fp16 N(0,1) scaled per (tensor, head) by U(0.01,0.02): "
                    "logits within a fraction of a unit, so every key keeps a non-zero e4m3 probability "
                    "(the dense-softmax case of the FP8 attention); LogScale"),
    "final_n8k_m1k_h8_gated": Workload(
        "final_n8k_m1k_h8_gated", 8192, 1024, 8, head_factor=(0.5, 4.0), gated=True, seed=6,
        description="N=8192, M=1024, H=8, d=64, fp16 N(0,1) scaled per (tensor, head) by U(0.5,4); "
                    "GatedLogScale; at most 8,192 context rows (or the final layer): normal-precision fp16 "
                    "attention"),
    "ragged_b16_n16k_m1k_h8": Workload(
        "ragged_b16_n16k_m1k_h8", 16384, 1024, 8, batch=16, ragged=(0.5, 1.0), seed=7,
        description="16 estimators in one batch, padded to N=16384 context rows, each with n_b ~ "
                    "U{8193..16384} unmasked rows; M=1024 queries, H=8, d=64, fp16 N(0,1); LogScale with "
                    "n = n_b; padding rows hold random values the layer must ignore"),
    "cached_n512k_m1k_h8": Workload(
        "cached_n512k_m1k_h8", 524288, 1024, 8, cached=True, seed=5,
        description="M=1024 fp16 N(0,1) queries, H=8, d=64, LogScale n=524288, against a resident FP8 "
                    "K/V cache of 524288 rows; equal across query batch splits 1/64/1024"),
}


def _normal_fill(out: np.ndarray, seed: int, tensor: str) -> None:
    flat = out.reshape(-1)
    n = flat.size
    tid = _TENSOR_IDS[tensor]

    def one(ci: int):
        lo, hi = ci * _CHUNK, min(n, (ci + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, ci])))
        flat[lo:hi] = g.standard_normal(hi - lo, dtype=np.float32)

    n_chunks = (n + _CHUNK - 1) // _CHUNK
    if n_chunks <= 2:
        for ci in range(n_chunks):
            one(ci)
    else:
        with ThreadPoolExecutor(max_workers=8) as ex:
            list(ex.map(one, range(n_chunks)))


def _outliers(x32: np.ndarray, seed: int, tensor_tid: int, frac: float, scale: float) -> None:
    flat = x32.reshape(-1)
    n = flat.size
    for ci in range((n + _CHUNK - 1) // _CHUNK):
        lo, hi = ci * _CHUNK, min(n, (ci + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TENSOR_IDS["outlier"], tensor_tid, ci])))
        mask = g.random(hi - lo) < frac
        flat[lo:hi][mask] *= np.float32(scale)


def _tensor(w: Workload, tensor: str, shape, seed: int) -> np.ndarray:
    x = np.empty(shape, np.float32)
    _normal_fill(x, seed, tensor)
    if w.head_factor is not None:
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TENSOR_IDS["head_factor"],
                                                                          _TENSOR_IDS[tensor]])))
        f = g.uniform(w.head_factor[0], w.head_factor[1], size=w.heads).astype(np.float32)
        x *= f.reshape((1,) * (len(shape) - 2) + (w.heads, 1))
    if w.outliers > 0:
        _outliers(x, seed, _TENSOR_IDS[tensor], w.outliers, w.outlier_scale)
    return x.astype(np.float16)


def make_inputs(w: Workload, seed: int | None = None, n_ctx: int | None = None, n_query: int | None = None,
                heads: int | None = None, batch: int | None = None) -> dict:
    """Host (numpy) inputs of a workload; sizes may be overridden for small cases.

    Returns q [B,T,H,d] (raw, before query scaling), k, v [B,N,H,d], c_h [H] fp32,
    gate [B,T,H] fp16 or None, plus the sizes.  For a cached workload the
    returned q holds the context rows of the fitted layer followed by the M
    prediction queries, drawn from a separate stream ("queries").
    """
    if any(a is not None for a in (n_ctx, n_query, heads, batch)):
        w = dataclasses.replace(w, n_ctx=n_ctx if n_ctx is not None else w.n_ctx,
                                n_query=n_query if n_query is not None else w.n_query,
                                heads=heads if heads is not None else w.heads,
                                batch=batch if batch is not None else w.batch)
    s = w.seed if seed is None else seed
    B, N, M, H, d = w.batch, w.n_ctx, w.n_query, w.heads, w.head_dim
    q = _tensor(w, "q", (B, N + M, H, d), s)
    k = _tensor(w, "k", (B, N, H, d), s)
    v = _tensor(w, "v", (B, N, H, d), s)
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([s, _TENSOR_IDS["c_h"]])))
    c_h = g.uniform(0.5, 1.5, size=H).astype(np.float32)
    gate = None
    if w.gated:
        gate = np.empty((B, N + M, H), np.float32)
        _normal_fill(gate, s, "gate")
        gate = gate.astype(np.float16)
    ctx_len = None
    if w.ragged is not None:
        lo = max(1, int(np.floor(w.ragged[0] * N)) + 1)
        hi = max(lo, int(np.floor(w.ragged[1] * N)))
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([s, _TENSOR_IDS["ctx_len"]])))
        ctx_len = g.integers(lo, hi + 1, size=B).astype(np.int64)
    out = dict(workload=w, q=q, k=k, v=v, c_h=c_h, gate=gate, B=B, N=N, M=M, H=H, d=d, ctx_len=ctx_len)
    if w.cached:
        qq = np.empty((B, M, H, d), np.float32)
        _normal_fill(qq, s, "queries")
        out["queries"] = qq.astype(np.float16)
    return out


# --- ragged grouped-query prefill (a second workload, bf16, head dim 128) ---------

@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    q_lens: tuple          # query tokens per sequence
    kv_lens: tuple         # key/value tokens per sequence (the queries are the last q_len of them)
    q_heads: int
    kv_heads: int
    head_dim: int = 128
    causal: bool = True
    seed: int = 0
    description: str = ""


PREFILL_WORKLOADS = {
    "gqa4_prefill_b2": PrefillWorkload(
        "gqa4_prefill_b2", (32, 64), (256, 1024), 16, 4, seed=11,
        description="2 sequences, query lengths 32/64, key/value lengths 256/1024, 16 query heads sharing "
                    "4 key/value heads, head dim 128, bf16 N(0,1); causal, queries aligned to the end"),
}


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (input preparation only)."""
    u = np.ascontiguousarray(x32, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def make_prefill_inputs(w: PrefillWorkload, seed: int | None = None, q_lens=None, kv_lens=None) -> dict:
    """Packed ragged inputs: q [sum q_len, Hq, d], k / v [sum kv_len, Hkv, d] as bf16 bits
    (uint16), with host indptr arrays (int64, B + 1 entries)."""
    s = w.seed if seed is None else seed
    q_lens = tuple(w.q_lens if q_lens is None else q_lens)
    kv_lens = tuple(w.kv_lens if kv_lens is None else kv_lens)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    kvo = np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int64)
    out = {}
    for name, rows, heads in (("q", int(qo[-1]), w.q_heads), ("k", int(kvo[-1]), w.kv_heads),
                              ("v", int(kvo[-1]), w.kv_heads)):
        x = np.empty((rows, heads, w.head_dim), np.float32)
        _normal_fill(x, s, name)
        out[name] = bf16_bits(x)
    out.update(qo_indptr=qo, kv_indptr=kvo, q_lens=q_lens, kv_lens=kv_lens, q_heads=w.q_heads,
               kv_heads=w.kv_heads, head_dim=w.head_dim, causal=w.causal, workload=w)
    return out
