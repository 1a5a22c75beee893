"""The benchmark's multi-rank host logic on CPU: world size 2, gloo backend.

Ranks time independent problems; the reported time is the max over ranks and
only rank 0 prints (the reference arm runs on rank 0 alone)."""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys, json, io, contextlib
sys.path.insert(0, sys.argv[1])
import torch
import bench
rank, world = bench.init_dist("gloo")
assert world == 2
got = bench.reduce_max(1.5 + rank, torch.device("cpu"))
bench.barrier(torch.device("cpu"))
buf = io.StringIO()
with contextlib.redirect_stdout(buf):
    if rank == 1:
        bench.run_reference(type("A", (), {"workload": "icl_n1k_m128_h4", "steps": 1, "warmup": 0, "cpu_rows": 4})())
print(json.dumps({"rank": rank, "max": got, "ref_out": buf.getvalue()}))
torch.distributed.destroy_process_group()
'''


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_max_over_ranks_and_rank0_output():
    port = _port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD, ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=240) for p in procs]
    import json
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e[-2000:]
    res = [json.loads(o.strip().splitlines()[-1]) for o, _ in outs]
    assert all(r["max"] == 2.5 for r in res)
    assert res[1]["ref_out"] == ""   # non-zero ranks print nothing in the reference arm


SHARD_CHILD = r'''
import os, sys, json
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import torch.distributed as dist
import oracle as orc
from fp8_quant_logscale_b200.sharded import shard_range
from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs

dist.init_process_group("gloo")
G, r = dist.get_world_size(), dist.get_rank()
N, M, H, B = 700, 45, 3, 2
inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=N, n_query=M, heads=H, batch=B)
c0, c1 = shard_range(N, G, r)
q0, q1 = shard_range(M, G, r)
rows = np.r_[c0:c1, N + q0:N + q1]
n_r = c1 - c0
# this rank's data only: its context rows and query rows of q (and gate), its rows of k, v
q_loc, g_loc = inp["q"][:, rows], inp["gate"][:, rows]
k_loc, v_loc = inp["k"][:, c0:c1], inp["v"][:, c0:c1]
# 1. query scaling with the global length, maxima over the local context rows
qs_loc = orc.qscale(np.ascontiguousarray(q_loc), N, inp["c_h"], np.ascontiguousarray(g_loc))
amax = torch.from_numpy(np.stack([np.abs(x[:, :n_r].astype(np.float32)).max(axis=(1, 3))
                                  for x in (qs_loc, k_loc, v_loc)]))
# 2. all-reduce(MAX)
dist.all_reduce(amax, op=dist.ReduceOp.MAX)
scales = (amax.numpy() / np.float32(448.0)).astype(np.float32)
scales[amax.numpy() == 0] = 1.0
# 3. codes of the local rows with the reduced scales
q8_loc = orc.quantize(qs_loc, scales[0])
k8_loc = orc.quantize(np.ascontiguousarray(k_loc), scales[1])
v8_loc = orc.quantize(np.ascontiguousarray(v_loc), scales[2])
# 4. all-gather of K8 / V8 (padded to the largest slice), assembled in row order
n_max = max(shard_range(N, G, g)[1] - shard_range(N, G, g)[0] for g in range(G))
pad = lambda x: torch.from_numpy(np.pad(x, ((0, 0), (0, 0), (0, n_max - n_r), (0, 0))))
gathered = []
for x in (k8_loc, v8_loc):
    parts = [torch.empty((B, H, n_max, 64), dtype=torch.uint8) for _ in range(G)]
    dist.all_gather(parts, pad(x))
    gathered.append(np.concatenate([p.numpy()[:, :, :shard_range(N, G, g)[1] - shard_range(N, G, g)[0]]
                                    for g, p in enumerate(parts)], axis=2))
k8, v8 = gathered
# 5. this rank's rows against all keys
o16, o, _ = orc.attention(q8_loc, k8, v8, scales[0], scales[1], scales[2])
# the one-process oracle, on the full data
ref = orc.layer(inp["q"], inp["k"], inp["v"], N, inp["c_h"], inp["gate"])
ok = dict(scales=bool((scales[0] == ref["s_q"]).all() and (scales[1] == ref["s_k"]).all()
                      and (scales[2] == ref["s_v"]).all()),
          k8=bool((k8 == ref["k8"]).all()), v8=bool((v8 == ref["v8"]).all()),
          q8=bool((q8_loc == ref["q8"][:, :, rows]).all()),
          out=bool((o == ref["out"][:, rows]).all() and (o16.view(np.uint16) == ref["out16"][:, rows].view(np.uint16)).all()),
          n_rows=int(rows.size))
print(json.dumps(ok))
dist.destroy_process_group()
'''


def test_sharded_split_reproduces_the_one_process_oracle():
    """World size 2 on gloo, the oracle doing each rank's compute: per-slice maxima
    all-reduced with MAX, per-slice codes all-gathered, and each rank's rows attended
    against the gathered cache reproduce the one-process oracle's scales, e4m3 codes
    and outputs bit for bit."""
    port = _port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", SHARD_CHILD, ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=240) for p in procs]
    import json
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e[-2000:]
    res = [json.loads(o.strip().splitlines()[-1]) for o, _ in outs]
    for r in res:
        assert all(r[k] for k in ("scales", "k8", "v8", "q8", "out")), res
    assert sum(r["n_rows"] for r in res) == 745


CACHED_CHILD = r'''
import os, sys, json
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import torch.distributed as dist
import oracle as orc
from fp8_quant_logscale_b200.sharded import shard_range
from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs

dist.init_process_group("gloo")
G, r = dist.get_world_size(), dist.get_rank()
N, M, H, B = 5000, 37, 2, 1
inp = make_inputs(WORKLOADS["cached_n512k_m1k_h8"], n_ctx=N, n_query=M, heads=H, batch=B)
qs = orc.qscale(inp["q"], N, inp["c_h"])
s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qs, inp["k"], inp["v"]))
k8, v8 = orc.quantize(inp["k"], s_k), orc.quantize(inp["v"], s_v)
q8 = orc.quantize(orc.qscale(inp["queries"], N, inp["c_h"]), s_q)
L = orc.split_keys(N)
S = -(-N // L)
# this rank keeps only the keys of its chunks
c0, c1 = shard_range(S, G, r)
k0, k1 = c0 * L, min(c1 * L, N)
m, l, acc = orc.attention_partials(q8, k8[:, :, k0:k1], v8[:, :, k0:k1], s_q, s_k, N, L, c0, c1)
cmax = max(shard_range(S, G, g)[1] - shard_range(S, G, g)[0] for g in range(G))
def pad(x):
    out = np.full((cmax,) + x.shape[1:], -np.inf if x is m else 0.0)
    out[:x.shape[0]] = x
    return torch.from_numpy(out)
gathered = []
for x in (m, l, acc):
    parts = [torch.empty((cmax,) + x.shape[1:], dtype=torch.float64) for _ in range(G)]
    dist.all_gather(parts, pad(x))
    gathered.append(np.concatenate([p.numpy()[:shard_range(S, G, g)[1] - shard_range(S, G, g)[0]]
                                    for g, p in enumerate(parts)], axis=0))
got = orc.combine_partials(*gathered, s_v)
_, want, _ = orc.attention(q8, k8, v8, s_q, s_k, s_v, split=L)
print(json.dumps({"chunks": int(c1 - c0), "S": int(S),
                  "rel": float(np.abs(got - want).max() / np.abs(want).max())}))
dist.destroy_process_group()
'''


def test_cached_chunk_split_reproduces_the_one_process_oracle():
    """World size 2 on gloo, the oracle doing each rank's compute: each rank keeps only the keys
    of its split-KV chunks and computes their partial states; all-gathered and combined in chunk
    order they give the one-process oracle's cached prediction (to double rounding)."""
    port = _port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", CACHED_CHILD, ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=240) for p in procs]
    import json
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e[-2000:]
    res = [json.loads(o.strip().splitlines()[-1]) for o, _ in outs]
    assert sum(x["chunks"] for x in res) == res[0]["S"] >= 2
    assert all(x["rel"] <= 1e-12 for x in res), res
