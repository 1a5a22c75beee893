"""Pins of the oracle's context scales and e4m3 quantisation (CPU only).

Against: the definition's invariants (the amax element maps to +-448, nothing
exceeds it, scales come from context rows only, amax 0 gives scale 1, a
power-of-two rescaling of the input leaves the codes unchanged) and torch's
float8_e4m3fn cast of x / s (an independent RNE implementation).
"""
import numpy as np
import torch


def _x(B=2, rows=300, H=3, seed=0, scale=3.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, rows, H, 64)) * scale).astype(np.float16)


def test_scales_are_context_amax_over_448(orc):
    x = _x()
    n_ctx = 200
    s = orc.context_scales(x, n_ctx)
    a = np.abs(x[:, :n_ctx].astype(np.float32)).max(axis=(1, 3))
    assert (s == (a / np.float32(448.0)).astype(np.float32)).all()


def test_query_rows_do_not_change_scales(orc):
    x = _x()
    y = x.copy()
    y[:, 200:] *= np.float16(8)
    assert (orc.context_scales(x, 200) == orc.context_scales(y, 200)).all()


def test_amax_element_maps_to_448_and_queries_saturate(orc):
    x = _x()
    s = orc.context_scales(x, 200)
    x8 = orc.quantize(x, s)                       # [B,H,rows,d]
    dec = orc.e4m3_decode(x8)
    ctx = dec[:, :, :200]
    assert np.abs(ctx).max() == 448.0
    assert (np.abs(ctx).max(axis=(2, 3)) == 448.0).all()
    y = x.copy()
    y[:, 250] = np.float16(1000)                   # a query row far above the context amax
    y8 = orc.quantize(y, orc.context_scales(y, 200))
    assert (y8[:, :, 250] == 0x7E).all()


def test_zero_amax_gives_unit_scale(orc):
    x = np.zeros((1, 10, 2, 64), np.float16)
    s = orc.context_scales(x, 10)
    assert (s == 1.0).all()
    assert (orc.quantize(x, s) == 0).all()


def test_power_of_two_rescale_keeps_codes(orc):
    x = _x(scale=1.0)
    s1 = orc.context_scales(x, 300)
    s2 = orc.context_scales((x * np.float16(4)).astype(np.float16), 300)
    assert (s2 == s1 * 4).all()
    assert (orc.quantize(x, s1) == orc.quantize((x * np.float16(4)).astype(np.float16), s2)).all()


def test_matches_torch_cast(orc):
    x = _x(B=1, rows=2000, H=4, seed=5)
    s = orc.context_scales(x, 1500)
    got = orc.quantize(x, s)
    y = torch.from_numpy(x.astype(np.float32)) / torch.from_numpy(s).view(1, 1, -1, 1)
    y = y.clamp(-448, 448)
    want = y.to(torch.float8_e4m3fn).view(torch.uint8).permute(0, 2, 1, 3).contiguous().numpy()
    assert (got == want).all()
