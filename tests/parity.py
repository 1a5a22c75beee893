"""Shared parity gates for the GPU tests (test helper, imports the oracle only)."""
import numpy as np
import torch

# Output gates of the layer's specification, against the oracle on the same inputs.
MAX_ABS = 2e-2
MEAN_ABS = 1e-3
# Relative distance of a probability from an e4m3 rounding midpoint below which
# either neighbouring code is a correct result: it covers the kernel's
# hardware 2^x approximation and the tensor core's own fp32 accumulation order
# of the logits.  Outputs get the oracle's first-order allowance for exactly
# those keys and nothing more.
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


def gate(gpu_out, ref_out, allow, what=""):
    """Assert |gpu - oracle| <= max(MAX_ABS, 1 fp16 ulp of the value) + allowance
    elementwise, and mean |gpu - oracle| <= MEAN_ABS.  The output is fp16, so
    where one ulp exceeds MAX_ABS (|O| >= 64) rounding alone may take one ulp."""
    g = host(gpu_out).astype(np.float64) if isinstance(gpu_out, torch.Tensor) else gpu_out.astype(np.float64)
    d = np.abs(g - ref_out)
    excess = d - allow - np.maximum(0.0, fp16_ulp(ref_out) - MAX_ABS)
    strict = allow == 0
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()),
                 max_abs_strict=float(d[strict].max()) if strict.any() else 0.0,
                 allowed_frac=float((~strict).mean()), n=int(d.size))
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    assert excess.max() <= MAX_ABS, f"{what}: max |d| - allowance = {excess.max():.4g} > {MAX_ABS} ({stats})"
    assert d.mean() <= MEAN_ABS, f"{what}: mean |d| = {d.mean():.4g} > {MEAN_ABS} ({stats})"
    return stats
