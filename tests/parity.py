"""Shared parity gates for the GPU tests (test helper, imports the oracle only)."""
import numpy as np
import torch

# Output gates of the layer's specification, against the oracle on the same inputs.
MAX_ABS = 2e-2
MEAN_ABS = 1e-3
# Relative distance of a probability from an e4m3 rounding midpoint within which
# the oracle reports a key as ambiguous (an implementation whose probabilities
# err by that much may round it to the other code).  Reported only: the gate
# itself adds nothing for such keys.
DELTA = 1e-4


def dev(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host(t):
    return t.detach().cpu().numpy()


def fp16_ulp(x):
    """Spacing of fp16 values at |x| (2^-24 in the subnormal range)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.exp2(e - 10)


def gate(gpu_out, ref_out, allow=None, what=""):
    """Assert |gpu - oracle| <= max(MAX_ABS, 1 fp16 ulp of the oracle's value)
    elementwise and mean |gpu - oracle| <= MEAN_ABS.  The output is fp16, so where
    one ulp exceeds MAX_ABS (|O| >= 32) its rounding alone may take one ulp.

    `allow`, the oracle's ambiguity report, only enters the returned statistics:
    the share of outputs with an ambiguous key and the largest difference on the
    outputs without one."""
    g = host(gpu_out).astype(np.float64) if isinstance(gpu_out, torch.Tensor) else gpu_out.astype(np.float64)
    d = np.abs(g - ref_out)
    limit = np.maximum(MAX_ABS, fp16_ulp(ref_out))
    small = limit == MAX_ABS
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()),
                 margin=float(MAX_ABS - d[small].max()) if small.any() else MAX_ABS,
                 n=int(d.size))
    if allow is not None:
        clear = allow == 0
        stats["ambiguous_frac"] = float((~clear).mean())
        stats["max_abs_unambiguous"] = float(d[clear].max()) if clear.any() else 0.0
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    worst = np.unravel_index(np.argmax(d - limit), d.shape)
    assert (d <= limit).all(), (f"{what}: |d| = {d[worst]:.4g} > {limit[worst]:.4g} at {worst} "
                                f"(gpu {g[worst]!r}, oracle {ref_out[worst]!r}; {stats})")
    assert d.mean() <= MEAN_ABS, f"{what}: mean |d| = {d.mean():.4g} > {MEAN_ABS} ({stats})"
    return stats
