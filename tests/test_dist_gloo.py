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
