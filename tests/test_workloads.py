"""The seeded input generator: determinism, shapes and the stated distributions."""
import numpy as np

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs


def test_deterministic_and_seeded():
    w = WORKLOADS["icl_n1k_m128_h4"]
    a, b = make_inputs(w), make_inputs(w)
    assert all((a[k] == b[k]).all() for k in ("q", "k", "v", "c_h"))
    c = make_inputs(w, seed=99)
    assert not (a["q"] == c["q"]).all()


def test_shapes_and_distributions():
    w = WORKLOADS["icl_n16k_m1k_h8"]
    inp = make_inputs(w, n_ctx=4096, n_query=256)
    assert inp["q"].shape == (1, 4352, 8, 64) and inp["k"].shape == (1, 4096, 8, 64)
    assert inp["q"].dtype == np.float16 and inp["c_h"].dtype == np.float32
    assert ((inp["c_h"] >= 0.5) & (inp["c_h"] <= 1.5)).all()
    std = inp["k"].astype(np.float32).std(axis=(0, 1, 3))      # per head: U(0.5, 4) factors
    assert (std > 0.45).all() and (std < 4.2).all() and std.max() / std.min() > 1.5


def test_outliers_and_gate():
    w = WORKLOADS["icl_n128k_m1k_h8_gated"]
    inp = make_inputs(w, n_ctx=8192, n_query=128)
    k = np.abs(inp["k"].astype(np.float32))
    assert 0.0004 < (k > 8).mean() < 0.002         # ~0.1% of elements x20
    assert inp["gate"].shape == (1, 8320, 8) and abs(inp["gate"].astype(np.float32).std() - 1) < 0.05


def test_cached_workload_has_separate_queries():
    w = WORKLOADS["cached_n512k_m1k_h8"]
    inp = make_inputs(w, n_ctx=1024, n_query=64)
    assert inp["queries"].shape == (1, 64, 8, 64)
    assert not (inp["queries"] == inp["q"][:, 1024:]).all()
