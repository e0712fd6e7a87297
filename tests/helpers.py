"""Shared test helpers: error metrics, the parity report, and oracle runs on
chosen heads."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Pass criteria: max |x - ref| / max |ref| per output tensor, for bf16 inputs
# with fp32 state, and for the all-fp32 path.
TOL_BF16 = 2e-2
TOL_F32 = 1e-4

# (case, tensor, max |x - ref| / max |ref|, max elementwise |x - ref| / (|ref| +
# 1e-3 max |ref|)), appended by the parity tests; conftest.py prints it.
PARITY_REPORT: list = []


def _f64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, np.float64)


def rel_err(x, ref) -> float:
    x, ref = _f64(x), _f64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.isfinite(x).all(), "non-finite values"
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / max(den, 1e-30))


class ErrAccum:
    """max |x - ref| / max |ref| and the elementwise figure over a tensor
    compared in pieces (the pieces share one max |ref|, taken over all of
    them)."""

    def __init__(self):
        self.num = 0.0
        self.den = 0.0
        self.elem = []  # (|x - ref|, |ref|) maxima per piece, resolved at the end

    def add(self, x, ref):
        x, ref = _f64(x), _f64(ref)
        assert x.shape == ref.shape, (x.shape, ref.shape)
        assert np.isfinite(x).all(), "non-finite values"
        d = np.abs(x - ref)
        a = np.abs(ref)
        self.num = max(self.num, float(d.max(initial=0.0)))
        self.den = max(self.den, float(a.max(initial=0.0)))
        self.elem.append((d, a) if d.size <= (1 << 22) else self._reduce(d, a))

    @staticmethod
    def _reduce(d, a):
        # The final floor 1e-3 max|ref| is at least this piece's own floor, so
        # the elementwise maximum comes, in practice, from the entries that are
        # largest at the piece's floor or largest in absolute error: keep those.
        d, a = d.ravel(), a.ravel()
        r = d / (a + 1e-3 * a.max(initial=0.0) + 1e-300)
        keep = np.unique(np.concatenate([np.argpartition(d, -4096)[-4096:],
                                         np.argpartition(r, -4096)[-4096:]]))
        return d[keep], a[keep]

    def result(self):
        floor = 1e-3 * self.den
        elem = max((float((d / (a + floor)).max(initial=0.0)) for d, a in self.elem),
                   default=0.0)
        return self.num / max(self.den, 1e-30), elem


def record(case: str, tensor: str, x=None, ref=None, acc: ErrAccum | None = None):
    """Compute and keep the two error figures of one output tensor; returns
    the pass metric (max |x - ref| / max |ref|)."""
    if acc is None:
        acc = ErrAccum()
        acc.add(x, ref)
    rel, elem = acc.result()
    PARITY_REPORT.append((case, tensor, rel, elem))
    return rel


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
