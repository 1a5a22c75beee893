"""Pins of the oracle's FP8 attention and cached (split-KV) prediction (CPU only).

The oracle's attention is the layer's definition in double precision (logits of
the e4m3 Q and K times s_q s_k / sqrt(d), online softmax over 128-key tiles, P
rounded to e4m3 against the running maximum before P.V).  It is pinned against:
a naive full-row double softmax (quantisation of P switched off); a
materialised-P restatement in numpy with torch's e4m3 decode and an e4m3
rounding written here, over several tile sizes and split-KV chunkings; a
hand-worked golden example with exact powers of two; Q = 0 (mean of V);
constant V (the row sum normalises); permutation of the context rows; and
partitions of the query batch for the cached path.  The single-precision
diagnostic arithmetic is pinned by its own materialised version.
"""
import os

import numpy as np
import pytest
import torch

from fp8_quant_logscale_b200.workloads import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LOG2E = 1.4426950408889634


def _codes(orc, B, H, rows, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((B, rows, H, 64)) * scale).astype(np.float16)
    s = orc.context_scales(x, rows)
    return orc.quantize(x, s), s


def _problem(orc, B=1, H=2, T=40, N=300, seed=0, qscale=0.4):
    q8, sq = _codes(orc, B, H, T, seed, 1.0)
    k8, sk = _codes(orc, B, H, N, seed + 1, 1.0)
    v8, sv = _codes(orc, B, H, N, seed + 2, 1.0)
    sq = (sq * np.float32(qscale)).astype(np.float32)  # moderate logits
    return q8, k8, v8, sq, sk, sv


def _naive(orc, q8, k8, v8, sq, sk, sv):
    q = orc.e4m3_decode(q8) * sq[..., None, None]
    k = orc.e4m3_decode(k8) * sk[..., None, None]
    v = orc.e4m3_decode(v8) * sv[..., None, None]
    x = np.einsum("bhtd,bhnd->bhtn", q, k) / 8.0
    x -= x.max(-1, keepdims=True)
    p = np.exp(x)
    o = np.einsum("bhtn,bhnd->bhtd", p, v) / p.sum(-1)[..., None]
    return o.transpose(0, 2, 1, 3)  # [B,T,H,d]


@pytest.mark.parametrize("bc", [1, 7, 128, 300])
def test_unquantised_p_matches_naive_softmax(orc, bc):
    q8, k8, v8, sq, sk, sv = _problem(orc)
    _, out, _ = orc.attention(q8, k8, v8, sq, sk, sv, bc=bc, quant_p=False)
    ref = _naive(orc, q8, k8, v8, sq, sk, sv)
    assert np.abs(out - ref).max() <= 1e-5 * np.abs(ref).max() + 1e-7


def test_exact_reference_matches_naive(orc):
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 9, 3, 64)).astype(np.float16)
    k = rng.standard_normal((2, 20, 3, 64)).astype(np.float16)
    v = rng.standard_normal((2, 20, 3, 64)).astype(np.float16)
    got = orc.attention_exact(q, k, v)
    qd, kd, vd = (a.astype(np.float64).transpose(0, 2, 1, 3) for a in (q, k, v))
    x = qd @ kd.transpose(0, 1, 3, 2) / 8.0
    p = np.exp(x - x.max(-1, keepdims=True))
    want = ((p @ vd) / p.sum(-1)[..., None]).transpose(0, 2, 1, 3)
    assert np.abs(got - want).max() < 1e-12


def test_golden_worked_example(orc):
    lines = {ln.split()[0]: ln.split()[1:] for ln in open(os.path.join(GOLDEN, "softmax_worked_example.txt"))
             if ln.strip() and ln[0] != "#"}
    k2 = np.float32(LOG2E / 8.0)
    sk = np.float32(1.0) / k2
    for cand in (sk, np.nextafter(sk, np.float32(0)), np.nextafter(sk, np.float32(1e9))):
        if np.float32(np.float32(1.0) * cand) * k2 == np.float32(1.0):
            sk = cand
            break
    assert np.float32(sk * k2) == np.float32(1.0)
    q8 = np.full((1, 1, 1, 64), 0x38, np.uint8)
    k8 = np.stack([np.full(64, c, np.uint8) for c in (0x00, 0x08, 0x10)])[None, None]
    v8 = np.stack([np.full(64, c, np.uint8) for c in (0x38, 0x40, 0x48)])[None, None]
    one = np.ones((1, 1), np.float32)
    want = float(lines["out"][0])
    # in the definition the logit of key j is z_j * s_k / 8 = z_j * ln2 * (1 + eps), with eps the
    # distance of the fp32 s_k from 8 / log2(e): the probabilities 2^(-2(1+eps)), 2^(-(1+eps)), 1
    # still round to the e4m3 values 1/4, 1/2, 1, but a running-sum rescale exp(m - m') is 1/2 or
    # 1/4 only to within 2 ln2 |eps| relative
    eps = abs(float(sk) * LOG2E / 8.0 - 1.0)
    assert eps < 2.0 ** -22
    for bc in (1, 2, 128):
        # with every key in one tile O is exactly 3; with smaller tiles within the rescale error
        o16, o, _ = orc.attention(q8, k8, v8, one, np.full((1, 1), sk, np.float32), one, bc=bc)
        tol = 0.0 if bc >= 3 else 4.0 * np.log(2.0) * eps * want
        assert (np.abs(o - want) <= tol).all(), (bc, o[0, 0, 0, :4])
        assert (o16.astype(np.float64) == 3.0).all()
        # the single-precision diagnostic arithmetic lands on the same powers of two exactly
        o16, o, _ = orc.attention(q8, k8, v8, one, np.full((1, 1), sk, np.float32), one, bc=bc, arith="fp32")
        assert (o == want).all(), (bc, o[0, 0, 0, :4])


@pytest.mark.parametrize("bc", [7, 128])
def test_zero_query_gives_mean_of_v(orc, bc):
    _, k8, v8, sq, sk, sv = _problem(orc)
    q8 = np.zeros((1, 2, 5, 64), np.uint8)
    o16, o, _ = orc.attention(q8, k8, v8, sq, sk, sv, bc=bc)
    mean = orc.e4m3_decode(v8).mean(axis=2) * sv[..., None]      # [B,H,d]
    assert np.allclose(o, mean[:, None, :, :], rtol=1e-12, atol=1e-15)
    assert (o16.view(np.uint16) == orc.f16_encode(np.broadcast_to(mean[:, None], o.shape))).all()


def test_constant_v_normalises_to_one(orc):
    q8, k8, _, sq, sk, _ = _problem(orc)
    v8 = np.full_like(k8, 0x38)
    sv = np.ones_like(sq)
    o16, o, _ = orc.attention(q8, k8, v8, sq, sk, sv, bc=16)
    assert np.abs(o - 1.0).max() < 1e-14
    assert (o16.astype(np.float64) == 1.0).all()


def _e4m3_round(p):
    """Nearest e4m3 value of p >= 0 (ties to even), for p <= 448: binade spacing
    2^(e-3), subnormal spacing 2^-9.  Written here from the format, independent of
    the oracle's codec."""
    p = np.asarray(p, np.float64)
    _, e = np.frexp(p)                       # p in [2^(e-1), 2^e)
    step = np.exp2(np.maximum(e - 1, -6) - 3)
    return np.rint(p / step) * step          # p / step is exact; rint ties to even


def _torch_e4m3_decode(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _materialised_definition(q8, k8, v8, sq, sk, sv, bc, split=0):
    """The whole P matrix at once: x = z s_q s_k / 8 with z exact, the running maximum
    at each key's tile (restarting at every split chunk), P8 = e4m3(exp(x - run)),
    each key weighted by exp(run - M) against the row's overall maximum M."""
    q, k, v = (_torch_e4m3_decode(c) for c in (q8, k8, v8))     # [B,H,*,d]
    B, H, T, _ = q.shape
    N = k.shape[2]
    x = (q @ k.transpose(0, 1, 3, 2)) * (sq.astype(np.float64) * sk.astype(np.float64) / 8.0)[..., None, None]
    chunk = split if split > 0 else N
    run = np.empty_like(x)
    for c0 in range(0, N, chunk):
        m = np.full(x.shape[:-1], -np.inf)
        for j0 in range(c0, min(N, c0 + chunk), bc):
            j1 = min(j0 + bc, c0 + chunk, N)
            m = np.maximum(m, x[..., j0:j1].max(-1))
            run[..., j0:j1] = m[..., None]
    M = x.max(-1, keepdims=True)
    w = _e4m3_round(np.exp(x - run)) * np.exp(run - M)
    o = (w @ v) / w.sum(-1, keepdims=True) * sv[..., None, None]
    return o.transpose(0, 2, 1, 3)


@pytest.mark.parametrize("bc,split", [(200, 0), (128, 0), (7, 0), (32, 96), (128, 128)])
def test_materialised_p_matches_online(orc, bc, split):
    """The online oracle (tile by tile, rescaling at every new maximum, chunks combined
    in order) against the materialised restatement: the same e4m3 codes, sums equal to
    double rounding."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=24, N=200, seed=7, qscale=1.0)
    want = _materialised_definition(q8, k8, v8, sq, sk, sv, bc, split)
    _, out, _ = orc.attention(q8, k8, v8, sq, sk, sv, bc=bc, split=split)
    assert np.abs(out - want).max() <= 1e-12 * np.abs(want).max()


def test_materialised_p_finds_a_tile_error(orc):
    """The materialised restatement tells tile sizes apart on these inputs, so the pin
    above would catch a wrong tile boundary or a missed rescale."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=24, N=200, seed=7, qscale=1.0)
    a = _materialised_definition(q8, k8, v8, sq, sk, sv, 128)
    b = _materialised_definition(q8, k8, v8, sq, sk, sv, 7)
    assert np.abs(a - b).max() > 1e-6


def test_materialised_p_matches_online_fp32_diagnostic(orc):
    """The single-precision diagnostic: fp32 logits in e order, torch's e4m3 cast, one tile."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=24, N=200, seed=7, qscale=1.0)
    qf = orc.e4m3_decode(q8).astype(np.float32)
    kf = orc.e4m3_decode(k8).astype(np.float32)
    z = np.zeros((1, 2, 24, 200), np.float32)
    for e in range(64):
        z = (z + qf[..., e:e + 1] * kf[..., e][:, :, None, :]).astype(np.float32)
    c2 = (np.float32(sq * sk) * np.float32(LOG2E / 8.0)).astype(np.float32)[..., None, None]
    m2 = (z.max(-1, keepdims=True) * c2).astype(np.float32)
    t = (z.astype(np.float64) * c2.astype(np.float64) - m2.astype(np.float64)).astype(np.float32)
    p = np.exp2(t.astype(np.float64)).astype(np.float32)
    p8 = orc.e4m3_decode(torch.from_numpy(p).to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    vf = orc.e4m3_decode(v8)
    want = (np.einsum("bhtn,bhnd->bhtd", p8, vf) / p8.sum(-1)[..., None] * sv[..., None, None]).transpose(0, 2, 1, 3)
    _, out, allow = orc.attention(q8, k8, v8, sq, sk, sv, bc=200, delta=1e-6, arith="fp32")
    assert (np.abs(out - want) <= 1e-12 + allow).all()


def test_definition_and_fp32_arithmetic_agree_closely(orc):
    """The definition and the single-precision sequence give nearly the same outputs:
    their e4m3 probability codes differ only where a probability sits next to a
    rounding midpoint, and the rescale factors by fp32 rounding (relative 1e-6 here)."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=40, N=300, seed=29, qscale=1.0)
    _, a, allow = orc.attention(q8, k8, v8, sq, sk, sv, delta=1e-5)
    _, b, _ = orc.attention(q8, k8, v8, sq, sk, sv, arith="fp32")
    assert (np.abs(a - b) <= 1e-6 * np.abs(a).max() + allow).all()


def test_context_permutation(orc):
    q8, k8, v8, sq, sk, sv = _problem(orc, N=256, seed=11)
    perm = np.random.default_rng(0).permutation(256)
    _, o1, _ = orc.attention(q8, k8, v8, sq, sk, sv, bc=256)
    _, o2, _ = orc.attention(q8, k8[:, :, perm], v8[:, :, perm], sq, sk, sv, bc=256)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.abs(o1).max()
    # with several tiles each tile quantises P against its own running max, so a
    # permutation moves outputs by the e4m3 quantisation noise of P only
    _, o3, _ = orc.attention(q8, k8[:, :, perm], v8[:, :, perm], sq, sk, sv, bc=16)
    assert np.abs(o1 - o3).mean() < 3e-3 and np.abs(o1 - o3).max() < 5e-2


def test_cached_split_is_partition_invariant(orc):
    q8, k8, v8, sq, sk, sv = _problem(orc, T=33, N=700, seed=13)
    full16, full, _ = orc.attention(q8, k8, v8, sq, sk, sv, split=256)
    for part in (1, 5, 16):
        for r0 in range(0, 33, part):
            rows = np.arange(r0, min(33, r0 + part))
            o16, o, _ = orc.attention(q8, k8, v8, sq, sk, sv, rows=rows, split=256)
            assert (o == full[:, rows]).all()
            assert (o16.view(np.uint16) == full16[:, rows].view(np.uint16)).all()


def test_split_covering_all_keys_equals_one_pass(orc):
    q8, k8, v8, sq, sk, sv = _problem(orc, T=20, N=300, seed=17)
    a16, a, _ = orc.attention(q8, k8, v8, sq, sk, sv, split=0)
    b16, b, _ = orc.attention(q8, k8, v8, sq, sk, sv, split=512)
    assert (a == b).all() and (a16.view(np.uint16) == b16.view(np.uint16)).all()
    _, c, _ = orc.attention(q8, k8, v8, sq, sk, sv, split=128)
    assert np.abs(a - c).mean() < 3e-3 and np.abs(a - c).max() < 5e-2


def test_allowance_properties(orc):
    q8, k8, v8, sq, sk, sv = _problem(orc, seed=19)
    _, _, a0 = orc.attention(q8, k8, v8, sq, sk, sv, delta=0.0)
    _, _, a1 = orc.attention(q8, k8, v8, sq, sk, sv, delta=1e-4)
    _, _, a2 = orc.attention(q8, k8, v8, sq, sk, sv, delta=1e-2)
    _, _, a3 = orc.attention(q8, k8, v8, sq, sk, sv, delta=1e-4, kappa=1e-4)
    assert (a0 == 0).all() and (a1 >= 0).all() and (a2 >= a1).all() and a2.max() > 0 and (a3 >= a1).all()


_E4M3_POS = np.unique(_torch_e4m3_decode(np.arange(0x7F, dtype=np.uint8)))    # 0 .. 448, every value


def _flips(orc, q8, k8, v8, sq, sk, sv, bc, split, delta, kappa, n_random, seed):
    """Brute force on the materialised definition: for every (row, head), the keys whose
    probability lies within relative r_j = delta + kappa (|m2| + |t_j|) of an e4m3 midpoint
    (found here from the value grid, independently of the oracle); flip each alone, all of
    them together and random subsets to the other neighbouring code, and return the
    largest |O' - O| / allowance over all of them (must be <= 1)."""
    q, k, v = (_torch_e4m3_decode(c) for c in (q8, k8, v8))
    B, H, T, _ = q.shape
    N = k.shape[2]
    x = (q @ k.transpose(0, 1, 3, 2)) * (sq.astype(np.float64) * sk.astype(np.float64) / 8.0)[..., None, None]
    chunk = split if split > 0 else N
    run = np.empty_like(x)
    for c0 in range(0, N, chunk):
        m = np.full(x.shape[:-1], -np.inf)
        for j0 in range(c0, min(N, c0 + chunk), bc):
            j1 = min(j0 + bc, c0 + chunk, N)
            m = np.maximum(m, x[..., j0:j1].max(-1))
            run[..., j0:j1] = m[..., None]
    M = x.max(-1, keepdims=True)
    p = np.exp(x - run)
    val = _e4m3_round(p)
    idx = np.searchsorted(_E4M3_POS, val)
    below = _E4M3_POS[np.maximum(idx - 1, 0)]
    above = _E4M3_POS[np.minimum(idx + 1, _E4M3_POS.size - 1)]
    r = delta + kappa * (np.abs(run) + (run - x)) * LOG2E
    lo = (np.abs(p - (val + below) / 2) <= r * p) & (val > 0)
    hi = np.abs(p - (val + above) / 2) <= r * p
    alt = np.where(hi, above, np.where(lo, below, val))
    amb = lo | hi
    _, _, allow = orc.attention(q8, k8, v8, sq, sk, sv, bc=bc, split=split, delta=delta, kappa=kappa)
    allow = allow.transpose(0, 2, 1, 3)                                    # [B,H,T,d]
    scale = np.exp(run - M)
    o = ((val * scale) @ v) / (val * scale).sum(-1, keepdims=True)
    rng = np.random.default_rng(seed)
    worst, n_amb = 0.0, int(amb.sum())
    for b in range(B):
        for h in range(H):
            for i in range(T):
                keys = np.nonzero(amb[b, h, i])[0]
                if keys.size == 0:
                    continue
                sets = [[j] for j in keys] + [list(keys)]
                sets += [list(rng.choice(keys, rng.integers(1, keys.size + 1), replace=False))
                         for _ in range(n_random)]
                for S in sets:
                    w = val[b, h, i].copy()
                    w[S] = alt[b, h, i, S]
                    w *= scale[b, h, i]
                    o2 = (w @ v[b, h]) / w.sum()
                    d = np.abs(o2 - o[b, h, i]) * float(sv[b, h])
                    worst = max(worst, float((d / np.maximum(allow[b, h, i], 1e-300)).max()))
    return worst, n_amb


@pytest.mark.parametrize("bc,split,delta,kappa", [(200, 0, 2e-2, 0.0), (7, 0, 1e-2, 0.0), (32, 96, 3e-3, 1e-3),
                                                  (128, 0, 1e-3, 3e-3)])
def test_allowance_bounds_every_flip(orc, bc, split, delta, kappa):
    """The allowance is an upper bound on the output change of any set of ambiguous keys
    taking their other code (a large radius makes many keys ambiguous)."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=24, N=200, seed=31, qscale=1.0)
    worst, n_amb = _flips(orc, q8, k8, v8, sq, sk, sv, bc, split, delta, kappa, n_random=8, seed=1)
    assert n_amb > 100, n_amb
    assert worst <= 1.0, worst


def test_allowance_bounds_flips_of_keys_far_from_the_output(orc):
    """V rows around 3 with a third of them zero: flipping a key whose value is 0 moves O
    by its whole size, which the allowance's vmax term covers."""
    q8, k8, _, sq, sk, _ = _problem(orc, T=24, N=200, seed=37, qscale=3.0)
    rng = np.random.default_rng(41)
    v = (3.0 + 0.5 * rng.standard_normal((1, 200, 2, 64))).astype(np.float16)
    v[:, rng.random(200) < 0.33] = 0
    sv = orc.context_scales(v, 200)
    v8 = orc.quantize(v, sv)
    worst, n_amb = _flips(orc, q8, k8, v8, sq, sk, sv, 128, 0, 2e-2, 0.0, n_random=8, seed=2)
    assert n_amb > 100 and worst <= 1.0, (n_amb, worst)


def test_allowance_is_not_vacuous(orc):
    """The bound is within a factor 10 of a change some flip actually makes, so an
    allowance ten times too small would fail the brute force above."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=24, N=200, seed=31, qscale=1.0)
    worst, _ = _flips(orc, q8, k8, v8, sq, sk, sv, 200, 0, 2e-2, 0.0, n_random=0, seed=1)
    assert worst > 0.1, worst


def test_lossless_when_inputs_are_e4m3_values(orc):
    """Inputs that are exactly e4m3 values times 2^-6 quantise losslessly, so with P
    unquantised the scales -> codes -> attention chain equals exact attention."""
    rng = np.random.default_rng(23)
    def exact_e4m3_tensor(rows):
        c = rng.integers(0, 0x7E, size=(1, rows, 2, 64)).astype(np.uint8) | (rng.integers(0, 2, (1, rows, 2, 64)) << 7).astype(np.uint8)
        c[0, 0, :, 0] = 0x7E  # every head reaches 448 -> scale exactly 2^-6
        return (orc.e4m3_decode(c) * 2.0 ** -6).astype(np.float16)
    q, k, v = exact_e4m3_tensor(50), exact_e4m3_tensor(300), exact_e4m3_tensor(300)
    q = (q.astype(np.float32) * np.float32(0.125)).astype(np.float16)   # exact: power of two
    sq, sk, sv = (orc.context_scales(x, x.shape[1]) for x in (q, k, v))
    assert (sk == 2.0 ** -6).all() and (sv == 2.0 ** -6).all() and (sq == 2.0 ** -9).all()
    q8, k8, v8 = orc.quantize(q, sq), orc.quantize(k, sk), orc.quantize(v, sv)
    assert (orc.e4m3_decode(q8).transpose(0, 2, 1, 3) * 2.0 ** -9 == q.astype(np.float64)).all()
    _, out, _ = orc.attention(q8, k8, v8, sq, sk, sv, quant_p=False)
    exact = orc.attention_exact(q, k, v)
    assert np.abs(out - exact).max() <= 1e-5 * np.abs(exact).max()


@pytest.mark.parametrize("split,N", [(256, 700), (128, 300), (1024, 700)])
def test_chunk_partials_combine_to_the_chunked_attention(orc, split, N):
    """Every chunk's partial state, combined in chunk order, is the oracle's cached
    (chunked) attention; partials computed from a key slice equal those from all keys."""
    q8, k8, v8, sq, sk, sv = _problem(orc, T=21, N=N, seed=43, qscale=1.0)
    S = -(-N // split)
    m, l, acc = orc.attention_partials(q8, k8, v8, sq, sk, N, split, 0, S)
    got = orc.combine_partials(m, l, acc, sv)
    _, want, _ = orc.attention(q8, k8, v8, sq, sk, sv, split=split)
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()
    for c0, c1 in ((0, 1), (1, S), (S - 1, S)):
        if c1 <= c0:
            continue
        k0, k1 = c0 * split, min(c1 * split, N)
        ms, ls, accs = orc.attention_partials(q8, k8[:, :, k0:k1], v8[:, :, k0:k1], sq, sk, N, split, c0, c1)
        assert np.array_equal(ms, m[c0:c1]) and np.array_equal(ls, l[c0:c1]) and np.array_equal(accs, acc[c0:c1])
