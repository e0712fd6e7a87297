"""fp64 gradients of the KDA forward (test infrastructure only).

The forward is the token recurrence of Kimi Linear (aiwiki.ai), sections "Kimi
Delta Attention" and "The constrained DPLR form and the chunkwise algorithm":
per (sequence, head) S_t = (I - b_t k_t k_t^T) Diag(exp g_t) S_{t-1} +
b_t k_t v_t^T, o_t = S_t^T q_t.  Here it is written with plain PyTorch ops in
float64 on the CPU, token by token, and differentiated by autograd; the pages
give no backward equations.  Pinned (tests/test_backward_oracle.py) by central
finite differences of the C oracle (oracle.forward), an implementation this
module shares nothing with.  Small problems only: the loop is in Python.
"""
from __future__ import annotations

import numpy as np
import torch


def _t64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64)
    return torch.from_numpy(np.asarray(x, dtype=np.float64))


def forward_torch(q, k, v, g, beta, h0, cu_seqlens=None):
    """o [T, H, dv], final states [N, H, dk, dv] (float64 tensors, differentiable
    in every argument).  q, k, g [T, H, dk]; v [T, H, dv]; beta [T, H];
    h0 [N, H, dk, dv]; cu_seqlens [N + 1] (None: one sequence)."""
    T = q.shape[0]
    cu = [0, T] if cu_seqlens is None else [int(x) for x in cu_seqlens]
    outs, finals = [], []
    for s in range(len(cu) - 1):
        S = h0[s]  # [H, dk, dv]
        for t in range(cu[s], cu[s + 1]):
            Sbar = torch.exp(g[t])[:, :, None] * S
            w = torch.einsum("hcj,hc->hj", Sbar, k[t])
            u = beta[t][:, None] * (v[t] - w)
            S = Sbar + k[t][:, :, None] * u[:, None, :]
            outs.append(torch.einsum("hcj,hc->hj", S, q[t]))
        finals.append(S)
    o = torch.stack(outs) if outs else torch.zeros(0, *v.shape[1:], dtype=torch.float64)
    return o, torch.stack(finals)


def backward(q, k, v, g, beta, h0, do, dhT=None, cu_seqlens=None):
    """Gradients of sum(o * do) + sum(final_state * dhT) with respect to
    (q, k, v, g, beta, h0), as float64 numpy arrays in that order."""
    args = [_t64(x).requires_grad_(True) for x in (q, k, v, g, beta, h0)]
    o, hN = forward_torch(*args, cu_seqlens=cu_seqlens)
    loss = (o * _t64(do)).sum()
    if dhT is not None:
        loss = loss + (hN * _t64(dhT)).sum()
    grads = torch.autograd.grad(loss, args, allow_unused=True)
    return tuple(np.zeros(a.shape) if gr is None else gr.numpy() for a, gr in zip(args, grads))
