"""Shared test helpers: upload synthetic inputs, run the CUDA path through the
binding, compare against the oracle with the acceptance tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Acceptance tolerances against the oracle.
TOL_ROW = 2e-3          # per-row loss and lse, absolute
TOL_MEAN_REL = 1e-5     # mean loss, relative
TOL_GRAD = 1e-2         # dH, dE normwise relative, filtering off
TOL_GRAD_FILTER = 2e-2  # dH, dE normwise relative, filtering on
EPS_BF16 = 2.0 ** -12   # bf16 precision threshold of the gradient filter


def normwise(got: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(np.asarray(got, dtype=np.float64) - ref) / max(den, 1e-300))


def upload(x, dev="cuda"):
    """Inputs -> (H, segments-as-torch, y) on the GPU."""
    from linear_cross_entropy_cce_b200 import cce
    H = cce.bf16_from_bits(x.H, dev)
    segs = [(b, e, cce.bf16_from_bits(E, dev)) for b, e, E in x.segments]
    y = torch.from_numpy(x.y).to(dev)
    return H, segs, y


def run_fwd(x, H, segs, y, want_colmax=False, status=None):
    from linear_cross_entropy_cce_b200 import cce
    if len(segs) == 1 and segs[0][0] == 0 and segs[0][1] == x.wl.V:
        return cce.fwd(H, segs[0][2], y, x.ignore_index, want_colmax=want_colmax, status=status)
    return cce.fwd(H, None, y, x.ignore_index, segments=segs, V=x.wl.V,
                   want_colmax=want_colmax, status=status)


def run_bwd(x, H, segs, y, lse, dloss, **kw):
    from linear_cross_entropy_cce_b200 import cce
    if len(segs) == 1 and segs[0][0] == 0 and segs[0][1] == x.wl.V:
        dH, dE, dbg = cce.bwd(H, segs[0][2], y, lse, dloss, x.ignore_index, **kw)
        return dH, [dE], dbg
    return cce.bwd(H, None, y, lse, dloss, x.ignore_index, segments=segs, V=x.wl.V, **kw)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
