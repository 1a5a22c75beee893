"""Shared parity gates for the GPU tests (test helper, imports the oracle only)."""
import numpy as np
import torch

import oracle

# Output gates of the layer's specification, against the oracle on the same inputs.
MAX_ABS = 2e-2
MEAN_ABS = 1e-3

# Ambiguity radius of a key's e4m3 probability code (oracle.attention's delta and
# kappa) for the kernel's single-precision probabilities: the 2^x evaluation plus
# 32 fp32 roundings of the logit's size (see oracle.FP32_AMBIGUITY).  Where the
# definition's probability lies within that distance of a rounding midpoint,
# either neighbouring code is what a correct fp32 implementation may produce; the
# oracle's allowance bounds the output change of any such choice (pinned by
# brute-force flipping in tests/test_oracle_attention.py).
AMB = dict(oracle.FP32_AMBIGUITY)


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
    """Assert |gpu - oracle| <= max(MAX_ABS, 1 fp16 ulp of the oracle's value) + allow
    elementwise and mean |gpu - oracle| <= MEAN_ABS.  The output is fp16, so where one
    ulp exceeds MAX_ABS (|O| >= 32) its rounding alone may take one ulp.  `allow` is
    the oracle's ambiguity allowance: zero for every output none of whose keys sits
    within the AMB radius of an e4m3 midpoint, so there the raw limit holds."""
    g = host(gpu_out).astype(np.float64) if isinstance(gpu_out, torch.Tensor) else gpu_out.astype(np.float64)
    d = np.abs(g - ref_out)
    limit = np.maximum(MAX_ABS, fp16_ulp(ref_out))
    clear = allow == 0
    small = clear & (limit == MAX_ABS)
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()),
                 margin=float(MAX_ABS - d[small].max()) if small.any() else MAX_ABS,
                 max_abs_unambiguous=float(d[clear].max()) if clear.any() else 0.0,
                 ambiguous_frac=float((~clear).mean()),
                 allowance_used=int((d > limit).sum()), n=int(d.size))
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    worst = np.unravel_index(np.argmax(d - limit - allow), d.shape)
    assert (d <= limit + allow).all(), (f"{what}: |d| = {d[worst]:.4g} > {limit[worst]:.4g} + {allow[worst]:.4g} "
                                        f"at {worst} (gpu {g[worst]!r}, oracle {ref_out[worst]!r}; {stats})")
    assert d.mean() <= MEAN_ABS, f"{what}: mean |d| = {d.mean():.4g} > {MEAN_ABS} ({stats})"
    return stats
