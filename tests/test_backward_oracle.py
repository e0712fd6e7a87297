"""Pins of the gradient oracle (oracle/backward.py): directional derivatives
against central finite differences of the C forward oracle, and the
per-token backward recurrence that the CUDA kernel implements, checked
against the oracle's gradients."""
import numpy as np
import pytest

import oracle
from oracle import backward as bwd


def _problem(seed, lens=(7, 5), H=2, dk=6, dv=5):
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
    return [q, k, v, g, beta, h0], cu, do, dhT


def _loss(args, cu, do, dhT):
    o, hN = oracle.forward(*args[:5], args[5], cu)
    return float((o * do).sum() + (hN * dhT).sum())


def test_gradients_match_finite_differences():
    args, cu, do, dhT = _problem(1)
    grads = bwd.backward(*args, do, dhT, cu)
    r = np.random.default_rng(2)
    eps = 1e-6
    for i, (a, gr) in enumerate(zip(args, grads)):
        for _ in range(3):
            d = r.normal(size=a.shape)
            plus = [x.copy() for x in args]
            minus = [x.copy() for x in args]
            plus[i] = a + eps * d
            minus[i] = a - eps * d
            fd = (_loss(plus, cu, do, dhT) - _loss(minus, cu, do, dhT)) / (2 * eps)
            an = float((gr * d).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (i, fd, an)


def _recurrent_backward(q, k, v, g, beta, h0, do, dhT, cu):
    """The per-token backward recurrence (the CUDA kernel's arithmetic),
    derived from the forward step S_bar = Diag(alpha) S_prev, w = S_bar^T k,
    u = beta (v - w), S = S_bar + k u^T, o = S^T q."""
    dq, dk, dv, dg = (np.zeros_like(x) for x in (q, k, v, g))
    db = np.zeros_like(beta)
    dh0 = np.zeros_like(h0)
    H = q.shape[1]
    for s in range(len(cu) - 1):
        for h in range(H):
            S = h0[s, h].copy()
            prev = []
            for t in range(cu[s], cu[s + 1]):
                prev.append(S.copy())
                Sb = np.exp(g[t, h])[:, None] * S
                u = beta[t, h] * (v[t, h] - Sb.T @ k[t, h])
                S = Sb + np.outer(k[t, h], u)
            dS = dhT[s, h].copy()
            for t in range(cu[s + 1] - 1, cu[s] - 1, -1):
                Sp = prev[t - cu[s]]
                a = np.exp(g[t, h])
                Sb = a[:, None] * Sp
                w = Sb.T @ k[t, h]
                u = beta[t, h] * (v[t, h] - w)
                St = Sb + np.outer(k[t, h], u)
                dS += np.outer(q[t, h], do[t, h])
                dq[t, h] = St @ do[t, h]
                du = dS.T @ k[t, h]
                dk[t, h] = dS @ u
                dv[t, h] = beta[t, h] * du
                db[t, h] = du @ (v[t, h] - w)
                dw = -beta[t, h] * du
                dSb = dS + np.outer(k[t, h], dw)
                dk[t, h] += Sb @ dw
                dg[t, h] = a * (dSb * Sp).sum(axis=1)
                dS = a[:, None] * dSb
            dh0[s, h] = dS
    return dq, dk, dv, dg, db, dh0


@pytest.mark.parametrize("seed", [3, 4])
def test_recurrent_backward_matches_the_oracle(seed):
    args, cu, do, dhT = _problem(seed, lens=(9, 0, 4), H=3, dk=5, dv=7)
    q, k, v, g, beta, h0 = args
    ref = bwd.backward(*args, do, dhT, cu)
    got = _recurrent_backward(q, k, v, g, beta, h0, do, dhT, cu)
    order = [0, 1, 2, 3, 4, 5]  # q k v g beta h0 vs dq dk dv dg db dh0
    for i, j in zip(order, [0, 1, 2, 3, 4, 5]):
        np.testing.assert_allclose(got[j], ref[i], rtol=1e-10, atol=1e-12)


def test_head_gate_gradient_is_the_channel_sum():
    """Gated DeltaNet: with the gate spread over the channels, the gradient of
    the per-(token, head) gate is the sum of the per-channel gradients --
    checked against central finite differences of the C forward oracle in the
    head gate itself."""
    args, cu, do, dhT = _problem(9, lens=(6, 4), H=2, dk=5, dv=3)
    r = np.random.default_rng(10)
    T, H, dk = args[3].shape
    gh = -np.log1p(np.exp(r.normal(size=(T, H))))
    spread = lambda x: np.repeat(x[:, :, None], dk, axis=2)  # noqa: E731
    args[3] = spread(gh)
    dg_head = bwd.backward(*args, do, dhT, cu)[3].sum(axis=2)
    eps = 1e-6
    for _ in range(3):
        d = r.normal(size=gh.shape)
        plus, minus = list(args), list(args)
        plus[3], minus[3] = spread(gh + eps * d), spread(gh - eps * d)
        fd = (_loss(plus, cu, do, dhT) - _loss(minus, cu, do, dhT)) / (2 * eps)
        an = float((dg_head * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)
