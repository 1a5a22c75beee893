"""The row-sharded layer call (sharded.py) and its entry points on one GPU.

sdm_context_amax and sdm_quantize_with_scales are compared bit for bit with the
oracle (maxima of |Q'|, |K|, |V| over a slice; scales amax/448; e4m3 codes).
The whole split runs with G ranks emulated as threads on one GPU, their two
collectives done on the host between kernel launches (no kernel waits on
another): every rank's output rows and its full FP8 cache must equal the
one-process layer's bit for bit.  Cached prediction with the keys split by
split-KV chunk over the ranks equals the one-GPU cached prediction bit for bit.
Both splits also run through a real NCCL process group of one rank (the only
size one GPU allows)."""
import threading

import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200 import binding, sharded
from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import dev, host

pytestmark = pytest.mark.gpu


def _abs_max(x, rows):
    """[B, H] fp32 max |x| over rows [0, rows) of x [B, R, H, 64] (exact)."""
    if rows == 0:
        return np.zeros((x.shape[0], x.shape[2]), np.float32)
    return np.abs(x[:, :rows].astype(np.float32)).max(axis=(1, 3))


@pytest.mark.parametrize("gated", [False, True])
def test_context_amax_and_quantize_with_scales(cuda_lib, orc, gated):
    N, M, H, B = 1500, 70, 3, 2
    inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated" if gated else "icl_n16k_m1k_h8"], n_ctx=N, n_query=M,
                      heads=H, batch=B)
    g = inp["gate"] if gated else None
    c0, c1 = 400, 1100                       # a slice of the context rows
    q_loc = np.ascontiguousarray(np.concatenate([inp["q"][:, c0:c1], inp["q"][:, N:N + M]], axis=1))
    g_loc = None if g is None else np.ascontiguousarray(np.concatenate([g[:, c0:c1], g[:, N:N + M]], axis=1))
    k_loc, v_loc = np.ascontiguousarray(inp["k"][:, c0:c1]), np.ascontiguousarray(inp["v"][:, c0:c1])
    n_r = c1 - c0
    amax = binding.context_amax(dev(q_loc), dev(k_loc), dev(v_loc), n_r, N, dev(inp["c_h"]), dev(g_loc))
    qs_loc = orc.qscale(q_loc, N, inp["c_h"], g_loc)                # query scaling with the global n = N
    want = np.stack([_abs_max(qs_loc, n_r), _abs_max(k_loc, n_r), _abs_max(v_loc, n_r)])
    assert (host(amax) == want).all()
    # with the full context's maxima, the slice's scales and codes are the one-process ones
    qs = orc.qscale(inp["q"], N, inp["c_h"], g)
    full = np.stack([_abs_max(qs, N), _abs_max(inp["k"], N), _abs_max(inp["v"], N)])
    q8, k8, v8t, scales = binding.quantize_with_scales(dev(q_loc), dev(k_loc), dev(v_loc), n_r, N, dev(full),
                                                       dev(inp["c_h"]), dev(g_loc), ld_k=n_r + 5)
    s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qs, inp["k"], inp["v"]))
    sc = host(scales)
    assert (sc[0] == s_q).all() and (sc[1] == s_k).all() and (sc[2] == s_v).all()
    assert (host(q8) == orc.quantize(qs_loc, s_q)).all()
    assert (host(k8)[:, :, :n_r] == orc.quantize(k_loc, s_k)).all()
    v8 = orc.quantize(v_loc, s_v)
    assert (host(v8t)[..., :n_r] == v8.transpose(0, 1, 3, 2)).all() and not host(v8t)[..., n_r:].any()


def test_empty_slice_gives_zero_maxima(cuda_lib):
    q = torch.zeros((1, 5, 2, 64), dtype=torch.float16, device="cuda")
    amax = binding.context_amax(q, None, None, 0, 100, torch.ones(2, device="cuda"))
    assert not amax.any()


class _ThreadComm:
    """G ranks as threads of one process on one GPU: the collectives meet on the host."""

    def __init__(self, world, rank, shared):
        self.world, self.rank, self.shared = world, rank, shared

    def _exchange(self, t):
        torch.cuda.synchronize()
        self.shared["slots"][self.rank] = t.clone()
        torch.cuda.synchronize()
        self.shared["barrier"].wait()
        got = torch.stack(self.shared["slots"])
        self.shared["barrier"].wait()
        return got

    def all_reduce_max_(self, t):
        t.copy_(self._exchange(t).amax(0))

    def all_gather(self, t):
        return self._exchange(t)


def _threads(G, fn):
    """fn(rank, comm) on G threads; returns the per-rank results."""
    shared = dict(barrier=threading.Barrier(G), slots=[None] * G)
    results, errors = [None] * G, []

    def rank_main(r):
        try:
            results[r] = fn(r, _ThreadComm(G, r, shared))
        except BaseException as e:   # noqa: BLE001 -- reported by the test thread
            errors.append(e)
            shared["barrier"].abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    return results


def _run_ranks(G, inp, gated):
    N, M = inp["N"], inp["M"]

    def rank_main(r, comm):
        c0, c1 = sharded.shard_range(N, G, r)
        q0, q1 = sharded.shard_range(M, G, r)
        rows = np.r_[c0:c1, N + q0:N + q1]
        q_loc = dev(np.ascontiguousarray(inp["q"][:, rows]))
        g_loc = dev(np.ascontiguousarray(inp["gate"][:, rows])) if gated else None
        out, cache = sharded.sharded_icl_attention(q_loc, dev(np.ascontiguousarray(inp["k"][:, c0:c1])),
                                                   dev(np.ascontiguousarray(inp["v"][:, c0:c1])), N, M,
                                                   dev(inp["c_h"]), comm, g_loc)
        torch.cuda.synchronize()
        return rows, host(out), host(cache.k8), host(cache.v8t), host(cache.scales)

    return _threads(G, rank_main)


@pytest.mark.parametrize("G,N,M,gated", [(2, 3000, 200, False), (3, 2049, 130, True), (4, 1000, 3, False),
                                         (8, 9000, 1024, False)])
def test_sharded_layer_equals_one_process(cuda_lib, G, N, M, gated):
    H, B = 4, 1
    inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated" if gated else "icl_n16k_m1k_h8"], n_ctx=N, n_query=M,
                      heads=H, batch=B)
    g = inp["gate"] if gated else None
    cache = cuda_lib.FP8Cache(B, N, H, "cuda")
    want = host(cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), dev(g),
                                       cache=cache))
    k8, v8t, sc = host(cache.k8), host(cache.v8t), host(cache.scales)
    for rows, out, rk8, rv8t, rsc in _run_ranks(G, inp, gated):
        assert np.array_equal(out.view(np.uint16), want[:, rows].view(np.uint16))
        assert np.array_equal(rk8, k8) and np.array_equal(rv8t, v8t) and np.array_equal(rsc, sc)


@pytest.mark.parametrize("G,N,M,ragged", [(2, 40000, 300, False), (3, 40000, 64, False), (5, 33000, 129, False),
                                          (5, 3000, 7, False), (3, 9000, 40, True)])
def test_sharded_cached_attention(cuda_lib, orc, G, N, M, ragged):
    """Cached prediction with the cache's keys split by split-KV chunk over G ranks (threads on
    one GPU; with N = 3000 the 3 chunks leave two of five ranks without keys): every rank's
    combined output equals cached_attention's bit for bit, and the oracle's chunked attention
    within the layer's gates."""
    from parity import AMB, gate
    H, B = 3, 2 if ragged else 1
    inp = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=N, n_query=M, heads=H, batch=B)
    lens = [N, N * 2 // 3 + 5] if ragged else None
    cache = cuda_lib.FP8Cache(B, N, H, "cuda")
    cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache,
                           ctx_len=lens)
    queries, c_h = dev(inp["queries"]), dev(inp["c_h"])
    want = host(cuda_lib.cached_attention(queries, cache, c_h))
    S = binding.split_count(N)

    def rank_main(r, comm):
        k8s, v8ts = sharded.cache_key_slice(cache, *sharded.shard_range(S, G, r))
        out = sharded.sharded_cached_attention(queries, cache, k8s, v8ts, c_h, comm)
        torch.cuda.synchronize()
        return host(out)

    for out in _threads(G, rank_main):
        assert np.array_equal(out.view(np.uint16), want.view(np.uint16))
    if not ragged:
        N_ = inp["N"]
        qs = orc.qscale(inp["q"], N_, inp["c_h"])
        s_q, s_k, s_v = (orc.context_scales(x, N_) for x in (qs, inp["k"], inp["v"]))
        q8 = orc.quantize(orc.qscale(inp["queries"], N_, inp["c_h"]), s_q)
        _, o, allow = orc.attention(q8, orc.quantize(inp["k"], s_k), orc.quantize(inp["v"], s_v), s_q, s_k, s_v,
                                    split=orc.split_keys(N_), **AMB)
        gate(want, o, allow, f"sharded cached G{G} N{N}")


NCCL_CHILD = r'''
import os, sys, datetime
sys.path.insert(0, sys.argv[1])
import numpy as np, torch, torch.distributed as dist
from fp8_quant_logscale_b200 import binding, sharded
from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
torch.cuda.set_device(0)
N, M, H = 5000, 300, 4
inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=N, n_query=M, heads=H)
d = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
out, cache = sharded.sharded_icl_attention(d(inp["q"]), d(inp["k"]), d(inp["v"]), N, M, d(inp["c_h"]),
                                           sharded.ProcessGroupComm(), d(inp["gate"]))
ref_cache = binding.FP8Cache(1, N, H, "cuda")
ref = binding.icl_attention(d(inp["q"]), d(inp["k"]), d(inp["v"]), N, d(inp["c_h"]), d(inp["gate"]), cache=ref_cache)
torch.cuda.synchronize()
ok = torch.equal(out.view(torch.int16), ref.view(torch.int16)) and torch.equal(cache.k8, ref_cache.k8) \
    and torch.equal(cache.v8t, ref_cache.v8t) and torch.equal(cache.scales, ref_cache.scales)
# cached prediction with the keys split by chunk (one rank holds them all)
qq = d(inp["q"][:, N - 100:N])
k8s, v8ts = sharded.cache_key_slice(cache, 0, binding.split_count(N))
pred = sharded.sharded_cached_attention(qq, cache, k8s, v8ts, d(inp["c_h"]), sharded.ProcessGroupComm())
ok = ok and torch.equal(pred.view(torch.int16), binding.cached_attention(qq, ref_cache, d(inp["c_h"])).view(torch.int16))
dist.destroy_process_group()
print("NCCL_OK" if ok else "NCCL_MISMATCH")
'''


def test_sharded_layer_over_a_real_nccl_group(cuda_lib):
    """The split through torch.distributed's NCCL backend (a one-rank group: this box has one
    GPU), in a child process: the all-reduce(MAX) and all-gather calls run for real and the
    result equals the one-process layer bit for bit."""
    import os
    import socket
    import subprocess
    import sys
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", NCCL_CHILD, root], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "NCCL_OK" in r.stdout, r.stdout[-2000:]


def test_new_entry_points_refuse_bad_arguments(cuda_lib):
    """Host-side checks before any work is enqueued: chunk ranges, slice pitches, row ranges,
    slice row counts."""
    import ctypes
    L = binding.lib()
    N, M, H = 3000, 8, 2
    inp = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=N, n_query=M, heads=H)
    cache = cuda_lib.FP8Cache(1, N, H, "cuda")
    cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache)
    S = binding.split_count(N)
    q, c_h = dev(inp["queries"]), dev(inp["c_h"])
    acc, ml = binding.partial_buffers(cache, M)
    k8s, v8ts = sharded.cache_key_slice(cache, 0, S)
    ws = cuda_lib.new_workspace(cuda_lib.workspace_size(binding.OP_CACHED_PARTIALS, 1, N, M, H), "cuda")
    P = ctypes.c_void_p
    stream = P(torch.cuda.current_stream().cuda_stream)

    def partials(c0, c1, ld=v8ts.shape[3]):
        return L.sdm_cached_partials(P(q.data_ptr()), 1, M, H, 64, ctypes.byref(cache.struct), P(k8s.data_ptr()),
                                     P(v8ts.data_ptr()), ld, c0, c1, P(c_h.data_ptr()), None, P(acc.data_ptr()),
                                     P(ml.data_ptr()), P(ws.data_ptr()), ws.numel(), stream)

    assert partials(0, S) == 0
    for c0, c1 in ((0, S + 1), (1, 1), (-1, 1), (2, 1)):
        assert partials(c0, c1) == 1, (c0, c1)                         # SDM_ERR_INVALID_ARG
    assert partials(0, S, ld=v8ts.shape[3] - 128) == 1                 # pitch below the slice's keys
    assert partials(0, S, ld=v8ts.shape[3] + 1) == 1                   # pitch not a multiple of 128
    assert L.sdm_cache_put_rows(ctypes.byref(cache.struct), P(k8s.data_ptr()), N, P(v8ts.data_ptr()),
                                v8ts.shape[3], 1, N, stream) == 1     # rows [1, N + 1) outside the cache
    amax = torch.zeros((3, 1, H), dtype=torch.float32, device="cuda")
    qq = dev(inp["q"])
    assert L.sdm_context_amax(P(qq.data_ptr()), P(qq.data_ptr()), P(qq.data_ptr()), 1, 10, 9, H, 64, N,
                              P(c_h.data_ptr()), None, P(amax.data_ptr()), stream) == 1   # q_rows < n_ctx
    torch.cuda.synchronize()
