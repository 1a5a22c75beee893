"""GPU parity on inputs built so that whole 128-key tiles hold only e4m3-zero
probabilities.

Every row shares one direction u with the keys of two "hot" tiles, so the row
maxima sit in those tiles and the other keys lie hundreds of log2 units below
them: their probabilities round to the e4m3 zero.  The FP8 attention kernel
skips the 2^x work of such tiles; these inputs make it take each branch of that
skip -- the first skipped tile (zeros stored), the skipped tiles after it
(nothing stored), a live tile after a run of skipped ones, a ragged last tile --
on the one-call path and on split-KV chunks (which restart the running max).
Outputs must match the oracle within the specification's gates, like any other
input.
"""
import numpy as np
import pytest

from parity import AMB, dev, gate, host

pytestmark = pytest.mark.gpu
LOG2E = 1.4426950408889634
HOT = (3, 9)


def _f16(x):
    return np.asarray(x, np.float32).astype(np.float16)


def _hot_tile_inputs(N=2000, M=160, H=2, seed=21):
    rng = np.random.default_rng(seed)
    T = N + M
    u = rng.choice([-1.0, 1.0], size=(H, 64))
    q = 2.0 * u[None, None] + 0.3 * rng.standard_normal((1, T, H, 64))
    k = 0.3 * rng.standard_normal((1, N, H, 64))
    for j in HOT:
        k[:, 128 * j:128 * (j + 1)] += 2.0 * u[None, None]
    v = rng.standard_normal((1, N, H, 64))
    return dict(q=_f16(q), k=_f16(k), v=_f16(v), c_h=np.ones(H, np.float32), B=1, N=N, M=M, H=H)


def _dead_warp_tiles(orc, inp, split):
    """[H, row warps, key tiles] bool: every row of a 32-row warp has the tile's
    largest logit more than 11.5 log2 units below its running max (a margin over
    the kernel's 10.0625), computed in float64 from the oracle's FP8 codes; key tiles
    restart their running max at every split-KV chunk boundary."""
    N = inp["N"]
    qs = orc.qscale(inp["q"], N, inp["c_h"])
    s_q, s_k = orc.context_scales(qs, N), orc.context_scales(inp["k"], N)
    q = orc.e4m3_decode(orc.quantize(qs, s_q))[0].astype(np.float64)      # [H, T, d]
    k = orc.e4m3_decode(orc.quantize(inp["k"], s_k))[0].astype(np.float64)
    T, n_tiles = q.shape[1], (N + 127) // 128
    out = []
    for h in range(inp["H"]):
        c2 = float(s_q[0, h]) * float(s_k[0, h]) * LOG2E / 8.0
        z = q[h] @ k[h].T                                                  # [T, N]
        zt = np.full((T, n_tiles * 128), -np.inf)
        zt[:, :N] = z
        tmax = zt.reshape(T, n_tiles, 128).max(axis=2)
        run = np.empty_like(tmax)
        for j in range(n_tiles):
            fresh = split and (j * 128) % split == 0
            run[:, j] = tmax[:, j] if (j == 0 or fresh) else np.maximum(run[:, j - 1], tmax[:, j])
        dead = (tmax - run) * c2 < -11.5
        w = T // 32
        out.append(dead[:w * 32].reshape(w, 32, n_tiles).all(axis=1))
    return np.array(out)


def test_zero_tiles_one_call(cuda_lib, orc):
    inp = _hot_tile_inputs()
    N, M, H = inp["N"], inp["M"], inp["H"]
    dead = _dead_warp_tiles(orc, inp, split=0)
    # the construction reaches every branch of the skip, in every row warp
    assert dead[:, :, HOT[0] + 1:HOT[1]].all(), "tiles between the hot ones are skipped"
    assert not dead[:, :, HOT[1]].any(), "the second hot tile is live again"
    assert dead[:, :, -1].all(), "the ragged last tile is skipped"
    cache = cuda_lib.FP8Cache(1, N, H, "cuda")
    ws = cuda_lib.new_workspace(cuda_lib.workspace_size(1, 1, N, M, H, keep_cache=True), "cuda")
    out = cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache,
                                 ws=ws)
    st, flags = cuda_lib.sync_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    ref = orc.layer(inp["q"], inp["k"], inp["v"], N, inp["c_h"], **AMB)
    stats = gate(host(out), ref["out"], ref["allow"], "zero tiles, one call")
    print(f"\nzero tiles one call: {stats}")


@pytest.mark.parametrize("n_pred", [160, 64])
def test_zero_tiles_split_kv(cuda_lib, orc, n_pred):
    """160 queries run on the two-tile kernel, 64 on the one-tile kernel of small batches."""
    inp = _hot_tile_inputs()
    N, M, H = inp["N"], inp["M"], inp["H"]
    split = orc.split_keys(N)
    dead = _dead_warp_tiles(orc, inp, split=split)
    # the second chunk starts fresh on a cold tile (live), then its hot tile raises the max
    first = split // 128
    assert not dead[:, :, first].any() and dead[:, :, HOT[1] + 1:].all()
    cache = cuda_lib.FP8Cache(1, N, H, "cuda")
    cuda_lib.icl_attention(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), N, dev(inp["c_h"]), cache=cache)
    queries = np.ascontiguousarray(inp["q"][:, N:N + n_pred])
    pred = host(cuda_lib.cached_attention(dev(queries), cache, dev(inp["c_h"])))
    qs = orc.qscale(inp["q"], N, inp["c_h"])
    s_q, s_k, s_v = (orc.context_scales(x, N) for x in (qs, inp["k"], inp["v"]))
    k8, v8 = orc.quantize(inp["k"], s_k), orc.quantize(inp["v"], s_v)
    qq = orc.quantize(orc.qscale(queries, N, inp["c_h"]), s_q)
    _, o, allow = orc.attention(qq, k8, v8, s_q, s_k, s_v, split=split, **AMB)
    stats = gate(pred, o, allow, f"zero tiles, split-KV, {n_pred} queries")
    print(f"\nzero tiles split-KV, {n_pred} queries: {stats}")


def _unit_c2_scale():
    """The fp32 s_k for which the kernel's c2 = fp32(s_q s_k) * fp32(log2(e)/8) is exactly 1 (s_q = 1),
    so a logit in base-2 units is the raw dot product z."""
    k2 = np.float32(LOG2E / 8.0)
    sk = np.float32(1.0) / k2
    for cand in (sk, np.nextafter(sk, np.float32(0)), np.nextafter(sk, np.float32(1e9))):
        if np.float32(cand * k2) == np.float32(1.0):
            return cand
    raise AssertionError("no fp32 scale gives c2 = 1")


def _key_row(ones, extra_code=None):
    """64 e4m3 codes: `ones` elements of 1.0 (0x38), optionally one extra code, the rest 0."""
    r = np.zeros(64, np.uint8)
    r[:ones] = 0x38
    if extra_code is not None:
        r[ones] = extra_code
    return r


@pytest.mark.parametrize("rows,split", [(5, False), (300, False), (5, True), (160, True)])
def test_skip_threshold_band(cuda_lib, orc, rows, split):
    """Logits placed around the skip threshold, with every query row q8 = 1.0 and c2 = 1
    (so t = z - m in base-2 units, m = 64 from key 0 in the first tile):
      tile 1: every key at t = -10.1015625, just below -10.0625: the warps skip it (zero codes);
      tile 2: one key at t = -9.8984375: P = 2^-9.9 > 2^-10 is computed and rounds to 2^-9;
      tile 3: one key at t = -10.03125: above the threshold, so computed, but P <= 2^-10
              rounds to the e4m3 zero.
    Other keys have t = -64.  The output must equal the oracle's bit for bit."""
    N = 512
    assert orc.e4m3_decode(np.uint8(0x9D)) == -0.1015625 and orc.e4m3_decode(np.uint8(0x1D)) == 0.1015625
    assert orc.e4m3_decode(np.uint8(0x90)) == -0.03125
    k8 = np.zeros((1, 1, N, 64), np.uint8)
    k8[0, 0, 0] = _key_row(64)                       # z = 64: the maximum
    k8[0, 0, 128:256] = _key_row(54, 0x9D)           # z = 53.8984375
    k8[0, 0, 256] = _key_row(54, 0x1D)               # z = 54.1015625
    k8[0, 0, 384] = _key_row(54, 0x90)               # z = 53.96875
    v8 = np.full((1, 1, N, 64), 0x48, np.uint8)      # 4.0: any wrongly live key shows
    v8[0, 0, 0], v8[0, 0, 256] = 0x38, 0x40          # 1.0 and 2.0
    sk = _unit_c2_scale()
    one = np.ones((1, 1), np.float32)
    s_k = np.full((1, 1), sk, np.float32)
    q8 = np.full((1, 1, rows, 64), 0x38, np.uint8)
    z = orc.e4m3_decode(k8[0, 0]).sum(axis=1)
    assert z[0] == 64 and (z[128:256] == 53.8984375).all() and z[256] == 54.1015625 and z[384] == 53.96875
    cache = cuda_lib.FP8Cache(1, N, 1, "cuda")
    cache.k8.copy_(dev(k8))
    v8t = np.zeros((1, 1, 64, cache.ld_v), np.uint8)
    v8t[..., :N] = v8.transpose(0, 1, 3, 2)
    cache.v8t.copy_(dev(v8t))
    cache.scales.copy_(dev(np.array([1.0, sk, 1.0], np.float32).reshape(3, 1, 1)))
    cache.struct.filled = 1
    out = host(cuda_lib.fp8_attention(dev(q8), cache, split=split))
    o16, o, _ = orc.attention(q8, k8, v8, one, s_k, one, split=orc.split_keys(N) if split else 0)
    assert np.array_equal(out.view(np.uint16), o16.view(np.uint16)), (out[0, 0, 0, :4], o[0, 0, 0, :4])
    # the live key at -9.9 contributed 2^-9 * 2.0, nothing else but key 0
    want = (1.0 + 2.0 ** -9 * 2.0) / (1.0 + 2.0 ** -9)
    assert np.allclose(o, want, rtol=1e-15)
