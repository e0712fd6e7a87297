"""The chunk-form backward equations the CUDA kernels implement, written out in
numpy fp64 and checked against the gradient oracle (oracle/backward.py, fp64
autograd of the token recurrence).  This pins the derivation -- the steps of
each kernel, including the reduction of T^T dT T^T to Y U^T -- independently of
the kernels' arithmetic: a dropped term, a wrong sign or a transposed operand
in the derivation fails here at 1e-10.

Chunk form: Kimi Linear (aiwiki.ai), "The constrained DPLR form and the
chunkwise algorithm"."""
import numpy as np
import pytest

from oracle import backward as bwd


def _chunk_backward(q, k, v, g, beta, h0, do, dhT, cu, C):
    """Per (sequence, head): the forward's chunk quantities, the forward chain,
    E and F, the reverse chain, then the per-chunk gradient steps."""
    dq, dk, dv, dg = (np.zeros_like(x) for x in (q, k, v, g))
    db, dh0 = np.zeros_like(beta), np.zeros_like(h0)
    H = q.shape[1]
    for s in range(len(cu) - 1):
        for h in range(H):
            chunks = [(a, min(a + C, cu[s + 1])) for a in range(cu[s], cu[s + 1], C)]
            ch = []
            for a, b in chunks:
                G = np.cumsum(g[a:b, h], axis=0)
                K, Q, V, B = k[a:b, h], q[a:b, h], v[a:b, h], beta[a:b, h]
                E = np.exp(G[:, None, :] - G[None, :, :])          # [r, i, c]
                Araw = np.tril(np.einsum("rc,ic,ric->ri", K, K, E), -1)
                A = B[:, None] * Araw
                P = np.tril(np.einsum("rc,ic,ric->ri", Q, K, E))
                Kt, Qt, Kb = K * np.exp(G), Q * np.exp(G), K * np.exp(G[-1] - G)
                IA = np.eye(b - a) + A
                W = np.linalg.solve(IA, B[:, None] * Kt)
                Ut = np.linalg.solve(IA, B[:, None] * V)
                Do = do[a:b, h]
                Ec = P.T @ Do                                       # E = P^T dO
                F = Qt.T @ Do - W.T @ Ec                            # F = Qt^T dO - W^T E
                ch.append(dict(G=G, K=K, Q=Q, V=V, B=B, E=E, Araw=Araw, IA=IA, Kt=Kt, Qt=Qt,
                               Kb=Kb, W=W, Ut=Ut, Do=Do, Ec=Ec, F=F))
            S = h0[s, h].copy()
            for c in ch:                                            # forward chain
                c["S"] = S.copy()
                c["U"] = c["Ut"] - c["W"] @ S
                S = np.exp(c["G"][-1])[:, None] * S + c["Kb"].T @ c["U"]
            dS = dhT[s, h].copy()
            for c in reversed(ch):                                  # reverse chain
                c["dSx"] = dS.copy()
                X = c["Kb"] @ dS
                c["dU"] = c["Ec"] + X
                dS = np.exp(c["G"][-1])[:, None] * dS - c["W"].T @ X + c["F"]
            dh0[s, h] = dS
            for (a, b), c in zip(chunks, ch):
                S, dSx, U, dU, B, G = c["S"], c["dSx"], c["U"], c["dU"], c["B"], c["G"]
                K, Q, E = c["K"], c["Q"], c["E"]
                Y = np.linalg.solve(c["IA"].T, dU)                  # Y = T^T dU
                dv[a:b, h] = B[:, None] * Y
                dA = -np.tril(Y @ U.T, -1)                          # = -T^T dT T^T, lower
                dP = np.tril(c["Do"] @ U.T)
                YS = Y @ S.T
                dQt, dKb = c["Do"] @ S.T, U @ dSx.T
                dKt = -B[:, None] * YS
                db[a:b, h] = ((Y * c["V"]).sum(1) + (dA * c["Araw"]).sum(1)
                              - (c["Kt"] * YS).sum(1))
                dAr = B[:, None] * dA
                rowA = np.einsum("ri,ic,ric->rc", dAr, K, E)
                colA = np.einsum("ri,rc,ric->ic", dAr, K, E)
                dQp = np.einsum("ri,ic,ric->rc", dP, K, E)
                colP = np.einsum("ri,rc,ric->ic", dP, Q, E)
                eG, eB = np.exp(G), np.exp(G[-1] - G)
                dq[a:b, h] = dQp + dQt * eG
                dk[a:b, h] = rowA + colA + colP + dKt * eG + dKb * eB
                dG = (K * (rowA - colA - colP) + Q * dQp + dQt * c["Qt"] + dKt * c["Kt"]
                      - dKb * c["Kb"])
                dG[-1] += (dKb * c["Kb"]).sum(0) + (S * dSx).sum(1) * np.exp(G[-1])
                dg[a:b, h] = np.cumsum(dG[::-1], axis=0)[::-1]
    return dq, dk, dv, dg, db, dh0


def _problem(seed, lens, H, dk, dv):
    r = np.random.default_rng(seed)
    T = sum(lens)
    q = r.normal(size=(T, H, dk))
    k = r.normal(size=(T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.normal(size=(T, H, dv))
    g = -np.log1p(np.exp(r.normal(size=(T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-r.normal(size=(T, H))))
    h0 = r.normal(size=(len(lens), H, dk, dv)) * 0.3
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    do = r.normal(size=(T, H, dv))
    dhT = r.normal(size=(len(lens), H, dk, dv))
    return q, k, v, g, beta, h0, do, dhT, cu


@pytest.mark.parametrize("C", [1, 4, 16])
def test_chunk_form_backward_matches_the_oracle(C):
    # several chunks per sequence, ragged tails, an empty sequence, dk != dv
    q, k, v, g, beta, h0, do, dhT, cu = _problem(40 + C, (37, 0, 20, 16), H=2, dk=8, dv=6)
    got = _chunk_backward(q, k, v, g, beta, h0, do, dhT, cu, C)
    ref = bwd.backward(q, k, v, g, beta, h0, do, dhT, cu)
    for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref):
        err = np.abs(x - r).max() / max(np.abs(r).max(), 1e-30)
        assert err <= 1e-10, (name, C, err)
