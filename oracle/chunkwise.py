"""fp64 restatement of the chunkwise (WY / UT) form of KDA -- test infrastructure.

Kimi Linear (aiwiki.ai), section "The constrained DPLR form and the chunkwise
algorithm": the sequence is split into chunks; inside a chunk the product of
the per-token Householder-like corrections is kept in a compact WY form, the
unit-triangular system is solved once (UT transform), and a state is carried
recurrently from chunk to chunk.  The pages give the idea but no equations; the
ones below are derived from the token recurrence

    S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t

by writing one step as ``S_r = Diag(a_r) S_{r-1} + k_r u_r^T`` with
``u_r = b_r (v_r - (Diag(a_r) S_{r-1})^T k_r)`` and unrolling inside a chunk
that starts from state ``S0``.  With ``G_r = sum_{j<=r} g_j`` (inclusive,
restarting at each chunk, per channel) and ``Gam_r = exp(G_r)``:

    A[r, i] = b_r * sum_c k[r,c] k[i,c] exp(G[r,c] - G[i,c])      (i < r)
    Tm      = (I + A)^{-1}                                          (UT transform)
    W       = Tm @ (diag(b) (K * Gam))           Ut = Tm @ (diag(b) V)
    U       = Ut - W @ S0
    P[r, i] = sum_c q[r,c] k[i,c] exp(G[r,c] - G[i,c])            (i <= r)
    O       = (Q * Gam) @ S0 + P @ U
    S_next  = Diag(Gam_L) S0 + (K * exp(G_L - G))^T @ U

(L = rows in the chunk; the last chunk of a sequence may be short.)  The
exponent differences are evaluated directly, never as a ratio of cumulative
decays.  This module is checked against the token recurrence in
``tests/test_oracle.py`` for several chunk sizes, including C = 1 where it
degenerates to the recurrence itself.
"""
from __future__ import annotations

import numpy as np


def chunk_step(q, k, v, g, b, S0):
    """One chunk for one head.  q, k, g: [L, dk]; v: [L, dv]; b: [L]; S0: [dk, dv].

    Returns a dict with the chunk's intermediates and results (all float64).
    """
    L, dk = k.shape
    G = np.cumsum(g, axis=0)
    D = G[:, None, :] - G[None, :, :]  # [r, i, c] = G_rc - G_ic
    E = np.exp(np.where(np.tril(np.ones((L, L), bool))[:, :, None], D, -np.inf))
    KK = np.einsum("rc,ic,ric->ri", k, k, E)
    A = np.tril(b[:, None] * KK, -1)
    Tm = np.linalg.inv(np.eye(L) + A)
    Gam = np.exp(G)
    W = Tm @ (b[:, None] * k * Gam)
    Ut = Tm @ (b[:, None] * v)
    U = Ut - W @ S0
    P = np.einsum("rc,ic,ric->ri", q, k, E)  # lower triangle incl. diagonal
    O = (q * Gam) @ S0 + P @ U
    S1 = Gam[-1][:, None] * S0 + (k * np.exp(G[-1][None, :] - G)).T @ U
    return dict(G=G, A=A, T=Tm, W=W, Ut=Ut, U=U, P=P, O=O, S_in=S0, S_out=S1)


def forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk: int = 64,
            keep=False):
    """Chunkwise forward; same conventions as :func:`oracle.forward` (flat [T, H, .]).

    If ``keep`` is true also returns a list, per (sequence, head, chunk) in
    order, of the intermediates of :func:`chunk_step`, keyed as
    ``(s, h, n)``.
    """
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    total, H, dk = q.shape
    dv = v.shape[-1]
    cu = np.array([0, total]) if cu_seqlens is None else np.asarray(cu_seqlens)
    N = len(cu) - 1
    o = np.zeros((total, H, dv))
    hN = np.zeros((N, H, dk, dv))
    inter = {}
    for s in range(N):
        for h in range(H):
            S = (np.zeros((dk, dv)) if initial_state is None
                 else np.asarray(initial_state[s, h], dtype=np.float64).copy())
            for n, t0 in enumerate(range(int(cu[s]), int(cu[s + 1]), chunk)):
                t1 = min(t0 + chunk, int(cu[s + 1]))
                r = chunk_step(q[t0:t1, h], k[t0:t1, h], v[t0:t1, h], g[t0:t1, h],
                               beta[t0:t1, h], S)
                o[t0:t1, h] = r["O"]
                S = r["S_out"]
                if keep:
                    inter[(s, h, n)] = r
            hN[s, h] = S
    if keep:
        return o, hN, inter
    return o, hN
