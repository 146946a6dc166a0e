"""Helpers that compare the CUDA path with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances of the ZeCO-path parity bar: max|delta| / max|ref| over a whole output tensor.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if hasattr(got, "detach") else np.asarray(got, np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref)) / (den if den > 0 else 1.0))


def forgetting_bound(log_g_slice) -> float:
    """max over (b, h, i) of the summed log-gate over a window: the log of the largest factor by
    which anything before the window can still reach the state after it."""
    s = log_g_slice.double().sum(dim=-2)
    return float(s.max())


def oracle_window(x, b, h, t0, t1, warm=8192, min_forget=-200.0):
    """Oracle outputs o[b, h, t0:t1] for a long sequence without replaying all of it.

    The oracle starts `warm` tokens before t0 from a zero state (from S0 when that reaches
    token 0).  The state the window receives then differs from the full-history state by a
    factor of at most exp(sum of log_g over the warm-up), asserted <= exp(min_forget) -- far
    below fp64 resolution -- so the window's reference is exact to double precision.
    """
    s = max(0, t0 - warm)
    sl = slice(s, t1)
    S0 = x.get("S0")
    if s > 0:
        fb = forgetting_bound(x["log_g"][b:b + 1, h:h + 1, s:t0])
        assert fb <= min_forget, f"warm-up too short to forget the prefix (bound {fb:.1f})"
        S0 = None
    elif S0 is not None:
        S0 = S0[b:b + 1, h:h + 1]
    o, _, _ = oracle.forward(x["q"][b:b + 1, h:h + 1, sl], x["k"][b:b + 1, h:h + 1, sl],
                             x["v"][b:b + 1, h:h + 1, sl], x["log_g"][b:b + 1, h:h + 1, sl], S0)
    return o[0, 0, t0 - s:]
