"""GPU parity of step 1 (fused LogScale / GatedLogScale) against the oracle:
bit-exact fp16 (the specification allows 1 ulp; both sides round identically)."""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs
from parity import dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,gated,n", [((1, 1152, 4), False, 1024), ((2, 77, 3), True, 1000),
                                           ((1, 5, 1), True, 1), ((3, 1, 128), False, 524288)])
def test_qscale_bit_exact(cuda_lib, orc, shape, gated, n):
    B, rows, H = shape
    rng = np.random.default_rng(rows)
    q = (rng.standard_normal((B, rows, H, 64)) * 3).astype(np.float16)
    c = rng.uniform(0.5, 1.5, H).astype(np.float32)
    g = (rng.standard_normal((B, rows, H)) * 2).astype(np.float16) if gated else None
    out = cuda_lib.qscale_fused(dev(q), dev(c), n, dev(g))
    torch.cuda.synchronize()
    want = orc.qscale(q, n, c, g)
    assert (host(out).view(np.uint16) == want.view(np.uint16)).all()


def test_qscale_in_place(cuda_lib, orc):
    inp = make_inputs(WORKLOADS["icl_n128k_m1k_h8_gated"], n_ctx=4096, n_query=100)
    q = dev(inp["q"])
    cuda_lib.qscale_fused(q, dev(inp["c_h"]), 4096, dev(inp["gate"]), out=q)
    torch.cuda.synchronize()
    want = orc.qscale(inp["q"], 4096, inp["c_h"], inp["gate"])
    assert (host(q).view(np.uint16) == want.view(np.uint16)).all()


def test_qscale_full_size_rows_sampled(cuda_lib, orc):
    """The 512K-context layer's query scaling on the device, checked on a row sample."""
    w = WORKLOADS["icl_n512k_m1k_h8"]
    inp = make_inputs(w)
    out = host(cuda_lib.qscale_fused(dev(inp["q"]), dev(inp["c_h"]), w.n_ctx))
    rows = np.random.default_rng(4).choice(w.rows, 2048, replace=False)
    want = orc.qscale(np.ascontiguousarray(inp["q"][:, rows]), w.n_ctx, inp["c_h"])
    assert (out[:, rows].view(np.uint16) == want.view(np.uint16)).all()
