"""Pins of the oracle's LogScale / GatedLogScale (CPU only).

Against: closed forms in double (q * c * ln n, and times 1 + tanh g) within the
rounding the eager chain allows; the special cases c*ln(n) = 1 (identity) and
g = 0 (gated == plain); and torch's own eager fp16 CPU ops performing the
unfused chain ("Fuse shared-length query scaling during inference", section
"Solution": every eager dtype-rounding boundary is preserved).
"""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs


def _inputs(B=2, rows=37, H=3, seed=0, gated=False):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((B, rows, H, 64)) * 2).astype(np.float16)
    c = rng.uniform(0.5, 1.5, H).astype(np.float32)
    g = rng.standard_normal((B, rows, H)).astype(np.float16) if gated else None
    return q, c, g


@pytest.mark.parametrize("n", [1, 7, 1024, 16384, 524288])
def test_logscale_closed_form(orc, n):
    q, c, _ = _inputs()
    got = orc.qscale(q, n, c).astype(np.float64)
    exact = q.astype(np.float64) * (c.astype(np.float64) * np.log(n)).reshape(1, 1, -1, 1)
    # two fp16 roundings (s_h and the product), each <= half an ulp relative
    tol = np.abs(exact) * 2.0 ** -10 * 1.001 + 2.0 ** -24
    assert (np.abs(got - exact) <= tol).all()


def test_gated_closed_form(orc):
    q, c, g = _inputs(gated=True)
    n = 4096
    got = orc.qscale(q, n, c, g).astype(np.float64)
    exact = (q.astype(np.float64) * (c.astype(np.float64) * np.log(n)).reshape(1, 1, -1, 1)
             * (1 + np.tanh(g.astype(np.float64)))[..., None])
    # relative roundings of s_h, q1 and q2 (half an ulp each), plus the absolute
    # roundings of u = fp16(tanh g) (<= 2^-12) and w = fp16(1 + u) (<= 2^-11),
    # which 1 + tanh g near 0 (g << 0) does not scale down: the eager fp16 chain
    # cancels there by construction.
    base = np.abs(q.astype(np.float64) * (c.astype(np.float64) * np.log(n)).reshape(1, 1, -1, 1))
    one_t = (1 + np.tanh(g.astype(np.float64)))[..., None]
    tol = base * (one_t * 3 * 2.0 ** -11 * 1.01 + 1.5 * 2.0 ** -11 * 1.01) + 2.0 ** -23
    assert (np.abs(got - exact) <= tol).all()


def test_identity_when_scale_is_one(orc):
    q, _, _ = _inputs()
    n = 1000
    lam = np.float32(orc.log_length(n))
    c = np.full(3, np.float32(1.0) / lam, np.float32)
    assert (np.float16(c[0] * lam) == np.float16(1.0))
    assert (orc.qscale(q, n, c).view(np.uint16) == q.view(np.uint16)).all()


def test_zero_gate_equals_logscale(orc):
    q, c, _ = _inputs()
    g = np.zeros(q.shape[:3], np.float16)
    assert (orc.qscale(q, 777, c, g).view(np.uint16) == orc.qscale(q, 777, c).view(np.uint16)).all()


def test_matches_torch_eager_chain(orc):
    """torch CPU fp16 ops, one op per eager step, give the same bits."""
    q, c, g = _inputs(B=1, rows=4096, H=4, seed=3, gated=True)
    n = 131072
    lam = torch.log(torch.tensor(float(n), dtype=torch.float32))
    assert abs(lam.item() - orc.log_length(n)) == 0.0
    s = (torch.from_numpy(c) * lam).to(torch.float16)            # per-head conversion
    qt = torch.from_numpy(q)
    q1 = qt * s.view(1, 1, -1, 1)                                  # fp16 * fp16 -> fp16
    plain = orc.qscale(q, n, c)
    assert (q1.numpy().view(np.uint16) == plain.view(np.uint16)).all()
    # gate: tanh rounded once to fp16 (double evaluation), then 1 + u and the multiply in fp16
    u = torch.from_numpy(np.tanh(g.astype(np.float64)).astype(np.float16))
    w = 1 + u
    q2 = q1 * w.unsqueeze(-1)
    gated = orc.qscale(q, n, c, g)
    assert (q2.numpy().view(np.uint16) == gated.view(np.uint16)).all()


def test_workload_inputs_go_through(orc):
    inp = make_inputs(WORKLOADS["icl_n1k_m128_h4"], n_ctx=256, n_query=16)
    out = orc.qscale(inp["q"], inp["N"], inp["c_h"])
    assert out.shape == inp["q"].shape and np.isfinite(out.astype(np.float32)).all()
