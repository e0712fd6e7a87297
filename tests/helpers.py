"""Shared test helpers: error metrics and oracle runs on chosen heads."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Pass criteria: max |x - ref| / max |ref| per output tensor, for bf16 inputs
# with fp32 state, and for the all-fp32 path.
TOL_BF16 = 2e-2
TOL_F32 = 1e-4


def rel_err(x, ref) -> float:
    x = x.detach().to("cpu", torch.float64).numpy() if isinstance(x, torch.Tensor) else \
        np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.isfinite(x).all(), "non-finite values"
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / max(den, 1e-30))


def tol_for(dtype: str) -> float:
    return TOL_BF16 if dtype == "bf16" else TOL_F32


def oracle_prefill(case, heads=None, threads=0):
    """Run the fp64 oracle on the case's (CPU) inputs, optionally on a subset of
    heads.  Returns (o [total, h, dv], final_state [N, h, dk, dv])."""
    sl = slice(None) if heads is None else list(heads)
    q, k, v, g, beta = (t[:, sl] for t in (case.q, case.k, case.v, case.g, case.beta))
    h0 = None if case.initial_state is None else case.initial_state[:, sl]
    cu = case.cu_host()
    return oracle.forward(q, k, v, g, beta, h0, cu_seqlens=cu, num_threads=threads)
