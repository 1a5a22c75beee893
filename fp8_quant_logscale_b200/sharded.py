"""One FP8 ICL attention layer call split over ranks, one process per GPU.

The layer's per-head scales come from all context rows ("[FP8 3/4] Integrate
FP8 attention and caching into TabICLv2", opening section: context-derived
scales), and every row attends to all context keys.  The pages run the layer on
one GPU and describe no multi-GPU scheme; this row split is the library's:

  rank r of G holds context rows [N r/G, N (r+1)/G) and query rows
  [M r/G, M (r+1)/G) of q (raw, before query scaling), and its context rows of
  k and v.
  1. sdm_context_amax over its context rows (query scaling with the global N);
  2. all-reduce(MAX) of the [3, B, H] fp32 maxima (12 B H bytes);
  3. sdm_quantize_with_scales of its rows: the scales are the same words on
     every rank, and equal to the one-process ones (a maximum is exact);
  4. all-gather of the K8 rows and V8^T columns (B H N 128 bytes in all) into
     rank-major buffers in this GPU's memory; sdm_cache_put_rows puts every
     rank's slice into a full FP8 cache;
  5. sdm_fp8_attention of its quantised rows (context, then query) against
     that cache.
A row's output depends only on its own e4m3 row, the full K8/V8 and the
scales, so each rank's rows equal the one-process layer's bit for bit.

Cached prediction can also be split by keys: with L = sdm_split_keys(N), the
cache's S = ceil(N / L) split-KV chunks are independent until their
fixed-order combine, so rank r keeps only the keys of chunks
[S r/G, S (r+1)/G) (cache_key_slice), computes their partials
(sdm_cached_partials), an all-gather brings every chunk's partials to every
rank, and sdm_cached_combine gives the one-GPU result bit for bit
(sharded_cached_attention).

Collectives go through a small interface (`all_reduce_max_`, `all_gather`):
`ProcessGroupComm` wraps a torch.distributed process group (NCCL on GPUs).
No kernel reads another GPU's memory.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as _b


def shard_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [lo, hi) of n that rank `rank` of `world` holds (contiguous, sizes differ by at most 1)."""
    return n * rank // world, n * (rank + 1) // world


class ProcessGroupComm:
    """The two collectives of the split, over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_reduce_max_(self, t: torch.Tensor) -> None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=self.group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[world, *t.shape]: every rank's t, in rank order (equal shapes on all ranks)."""
        out = torch.empty((self.world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=self.group)
        return out


def sharded_icl_attention(q_loc: torch.Tensor, k_loc: torch.Tensor, v_loc: torch.Tensor, n_ctx: int, n_query: int,
                          c_h: torch.Tensor, comm, gate_loc: torch.Tensor | None = None):
    """This rank's part of one FP8 layer call over comm.world ranks.

    q_loc [B, n_r + m_r, H, 64] fp16: the rank's context rows then its query rows,
    raw; k_loc, v_loc [B, n_r, H, 64]; gate_loc [B, n_r + m_r, H] or None; with
    (n_r, m_r) the sizes of shard_range(n_ctx / n_query, world, rank).
    Returns (out_loc [B, n_r + m_r, H, 64] fp16, cache): the rank's output rows and
    the full FP8 cache (every rank holds the same one, usable for cached prediction).
    """
    G, r = comm.world, comm.rank
    c0, c1 = shard_range(n_ctx, G, r)
    q0, q1 = shard_range(n_query, G, r)
    n_r, m_r = c1 - c0, q1 - q0
    B, T_r, H, d = q_loc.shape
    if T_r != n_r + m_r or (n_r > 0 and (k_loc.shape[1] != n_r or v_loc.shape[1] != n_r)):
        raise ValueError(f"rank {r}: q_loc must hold {n_r} + {m_r} rows and k_loc, v_loc {n_r}")
    dev = q_loc.device
    # 1-2: maxima of this rank's context rows, reduced over the ranks
    amax = _b.context_amax(q_loc, k_loc, v_loc, n_r, n_ctx, c_h, gate_loc)
    comm.all_reduce_max_(amax)
    # 3: scales (straight into the cache's scales block) and codes; the K8 planes and
    # V8^T rows are sized for the largest slice, so the all-gather moves equal buffers
    n_max = max(shard_range(n_ctx, G, g)[1] - shard_range(n_ctx, G, g)[0] for g in range(G))
    ld_v = max(_b.KV_TILE, -(-n_max // _b.KV_TILE) * _b.KV_TILE)
    cache = _b.FP8Cache(B, n_ctx, H, dev)
    cache.v8t.zero_()   # columns [N, ld_v) stay zero
    q8_loc, k8_loc, v8t_loc, _ = _b.quantize_with_scales(q_loc, k_loc, v_loc, n_r, n_ctx, amax, c_h, gate_loc,
                                                         ld_k=n_max, ld_v=ld_v, scales=cache.scales)
    # 4: every rank's slice into the full cache
    k_all = comm.all_gather(k8_loc)
    v_all = comm.all_gather(v8t_loc)
    for g in range(G):
        g0, g1 = shard_range(n_ctx, G, g)
        _b.cache_put_rows(cache, k_all[g], v_all[g], g0, g1 - g0)
    cache.struct.filled = 1
    # 5: this rank's rows against all keys
    out_loc = _b.fp8_attention(q8_loc, cache) if T_r > 0 else torch.empty((B, 0, H, d), dtype=torch.float16,
                                                                         device=dev)
    return out_loc, cache


def cache_key_slice(cache, c0: int, c1: int):
    """Copies of the keys of split-KV chunks [c0, c1) of a filled cache: K8 rows
    [B,H,n,64] and V8^T columns [B,H,64,ld] (ld a multiple of 128, zero past n)."""
    N = cache.n_ctx
    L = _b.split_keys(N)
    k0, k1 = c0 * L, min(c1 * L, N)
    ld = -(-(k1 - k0) // _b.KV_TILE) * _b.KV_TILE
    k8 = cache.k8[:, :, k0:k1].contiguous()
    v8t = torch.zeros((cache.batch, cache.heads, _b.HEAD_DIM, ld), dtype=torch.uint8, device=cache.k8.device)
    v8t[..., :k1 - k0].copy_(cache.v8t[..., k0:k1])
    return k8, v8t


def sharded_cached_attention(queries: torch.Tensor, cache, k8_slice: torch.Tensor, v8t_slice: torch.Tensor,
                             c_h: torch.Tensor, comm, gate: torch.Tensor | None = None) -> torch.Tensor:
    """Cached prediction of all M queries with the cache's keys split by chunk over the ranks.

    queries [B, M, H, 64] fp16 (the same on every rank); cache: the filled cache's
    descriptor (its scales block on this device; its K8 / V8^T are not read);
    k8_slice / v8t_slice: this rank's chunks [S r/G, S (r+1)/G) (cache_key_slice).
    Returns out [B, M, H, 64] fp16 on every rank, equal to cached_attention's bit for bit.
    """
    G, r = comm.world, comm.rank
    S = _b.split_count(cache.n_ctx)
    M = queries.shape[1]
    c0, c1 = shard_range(S, G, r)
    cmax = max(shard_range(S, G, g)[1] - shard_range(S, G, g)[0] for g in range(G))
    # room for G * cmax >= S chunks, so every rank's block [c0, c0 + cmax) lies inside
    acc, ml = _b.partial_buffers(cache, M, chunks=G * cmax)
    if c1 > c0:
        _b.cached_partials(queries, cache, k8_slice, v8t_slice, c0, c1, c_h, acc, ml, gate)
    acc_all = comm.all_gather(acc[c0:c0 + cmax])
    ml_all = comm.all_gather(ml[c0:c0 + cmax])
    full_acc, full_ml = _b.partial_buffers(cache, M)
    for g in range(G):
        g0, g1 = shard_range(S, G, g)
        full_acc[g0:g1].copy_(acc_all[g, :g1 - g0])
        full_ml[g0:g1].copy_(ml_all[g, :g1 - g0])
    return _b.cached_combine(full_acc, full_ml, cache, M)
