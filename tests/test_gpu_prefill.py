"""GPU parity of the ragged grouped-query prefill (sdm_gqa_prefill, bf16, head dim
128) against the oracle's double-precision attention of the same bf16 inputs.

Tolerance from the kernel's arithmetic: fp32 logits of 128 exact bf16 products
(error <= 128 * 2^-23 * sum_e |q_e k_e|), 2^x relative error < 3e-6,
probabilities rounded to bf16 for the P.V product (relative 2^-9) while the row
sum adds them unrounded, fp32 accumulation of O and l, one bf16 rounding of the
output.  Per (token, head), with S the largest sum_e |q_e k_e| over its visible
keys, n their count and c2 = log2(e)/sqrt(128):
    eta   = ln2 * c2 * S * 128 * 2^-23 + 3e-6
    bound = vmax * (2^-9 + 2 eta + (n/16 + n/8) 2^-23) + 1 bf16 ulp of |exact|
vmax being the largest |v| of the key/value head; the mean error must stay
within 1/16 of the mean bound.
"""
import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import PREFILL_WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu
C2 = 1.4426950408889634 / np.sqrt(128.0)
W = PREFILL_WORKLOADS["gqa4_prefill_b2"]


def bf16_ulp(x):
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def run(cuda_lib, inp, causal):
    out = cuda_lib.gqa_prefill(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), inp["qo_indptr"],
                               inp["kv_indptr"], causal=causal)
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


def check(cuda_lib, orc, inp, causal, what):
    Hq, Hkv = inp["q"].shape[1], inp["k"].shape[1]
    got = orc.bf16_decode(run(cuda_lib, inp, causal))
    exact = orc.gqa_prefill(inp["q"], inp["k"], inp["v"], inp["qo_indptr"], inp["kv_indptr"], Hq, Hkv, causal)
    q, k, v = (orc.bf16_decode(inp[x]) for x in ("q", "k", "v"))
    G = Hq // Hkv
    bound = np.zeros_like(exact)
    qo, kvo = inp["qo_indptr"], inp["kv_indptr"]
    for b in range(len(qo) - 1):
        q0, q1, k0, k1 = int(qo[b]), int(qo[b + 1]), int(kvo[b]), int(kvo[b + 1])
        nq, nk = q1 - q0, k1 - k0
        for h in range(Hq):
            g = h // G
            sa = np.abs(q[q0:q1, h]) @ np.abs(k[k0:k1, g]).T                       # [nq, nk]
            vis = (np.arange(nk)[None, :] <= (nk - nq + np.arange(nq))[:, None]) if causal else np.ones((nq, nk), bool)
            s_max = np.where(vis, sa, 0).max(axis=1)
            n = vis.sum(axis=1)
            eta = np.log(2.0) * C2 * s_max * 128 * 2.0 ** -23 + 3e-6
            vmax = np.abs(v[k0:k1, g]).max() if nk else 0.0
            bound[q0:q1, h] = (vmax * (2.0 ** -9 + 2 * eta + (n / 16 + n / 8) * 2.0 ** -23))[:, None]
    bound += bf16_ulp(exact)
    d = np.abs(got - exact)
    assert np.isfinite(got).all(), what
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()), max_ratio=float((d / bound).max()),
                 mean_bound=float(bound.mean()), n=int(d.size))
    print(f"\n{what}: {stats}")
    assert (d <= bound).all(), f"{what}: {stats}"
    assert d.mean() <= bound.mean() / 16, f"{what}: {stats}"


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_contract_shape(cuda_lib, orc, causal):
    """2 sequences, q 32/64, kv 256/1024, 16 query heads over 4 key/value heads."""
    check(cuda_lib, orc, make_prefill_inputs(W), causal, f"contract causal={causal}")


@pytest.mark.parametrize("q_lens,kv_lens", [((1, 17, 100), (1, 300, 1000)), ((5, 0, 33), (5, 7, 33)),
                                            ((129,), (129,)), ((40, 31), (2000, 31)),
                                            ((50, 3), (5000, 4200))])   # long key ranges
def test_prefill_ragged_lengths(cuda_lib, orc, q_lens, kv_lens):
    inp = make_prefill_inputs(W, q_lens=q_lens, kv_lens=kv_lens)
    check(cuda_lib, orc, inp, True, f"ragged q{q_lens} kv{kv_lens}")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (16, 2), (32, 2)])
def test_prefill_group_sizes(cuda_lib, orc, hq, hkv):
    import dataclasses
    w = dataclasses.replace(W, q_heads=hq, kv_heads=hkv)
    check(cuda_lib, orc, make_prefill_inputs(w, q_lens=(50, 13), kv_lens=(300, 13)), True, f"Hq{hq} Hkv{hkv}")


def test_prefill_many_sequences(cuda_lib, orc):
    """More sequences than one launch carries (64), lengths drawn at random."""
    rng = np.random.default_rng(7)
    q_lens = rng.integers(0, 40, size=70)
    kv_lens = q_lens + rng.integers(1, 200, size=70)
    check(cuda_lib, orc, make_prefill_inputs(W, q_lens=tuple(q_lens), kv_lens=tuple(kv_lens)), True, "70 sequences")


def test_prefill_is_deterministic_and_leaves_no_error(cuda_lib):
    inp = make_prefill_inputs(W)
    ws = cuda_lib.new_workspace(cuda_lib.gqa_prefill_workspace_size(inp["qo_indptr"], inp["kv_indptr"], 16, 4),
                                "cuda")
    a = cuda_lib.gqa_prefill(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), inp["qo_indptr"],
                             inp["kv_indptr"], ws=ws)
    b = cuda_lib.gqa_prefill(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), inp["qo_indptr"],
                             inp["kv_indptr"], ws=ws)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert cuda_lib.sync_status(ws) == (0, 0)


def test_prefill_workspace_reuse_across_batches(cuda_lib, orc):
    """One workspace for several different batches in a row."""
    shapes = [((50, 3), (5000, 4200)), ((1, 17, 100), (1, 300, 1000)), ((50, 3), (5000, 4200))]
    need = max(cuda_lib.gqa_prefill_workspace_size(np.concatenate([[0], np.cumsum(ql)]),
                                                   np.concatenate([[0], np.cumsum(kl)]), 16, 4) for ql, kl in shapes)
    ws = cuda_lib.new_workspace(need, "cuda")
    for ql, kl in shapes:
        inp = make_prefill_inputs(W, q_lens=ql, kv_lens=kl)
        got = cuda_lib.gqa_prefill(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), inp["qo_indptr"],
                                   inp["kv_indptr"], ws=ws)
        ref = cuda_lib.gqa_prefill(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), inp["qo_indptr"],
                                   inp["kv_indptr"])
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), (ql, kl)
    assert cuda_lib.sync_status(ws) == (0, 0)
