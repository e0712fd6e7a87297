"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: explicit
products of the dense transition matrices, special cases that reduce to other
named methods, an invariant, a hand-worked example, and composition rules.
Sources: Kimi Linear (aiwiki.ai), sections "Background: from the delta rule to
gated DeltaNet", "Kimi Delta Attention" and "The constrained DPLR form and the
chunkwise algorithm".
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import chunkwise

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, T, H, dk, dv, N=1, g_scale=1.0, with_h0=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, H, dk))
    k = r.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = r.standard_normal((T, H, dv))
    g = -np.log1p(np.exp(r.standard_normal((T, H, dk)))) * g_scale
    beta = 1 / (1 + np.exp(-r.standard_normal((T, H))))
    h0 = r.standard_normal((N, H, dk, dv)) if with_h0 else None
    return q, k, v, g, beta, h0


def _close(a, b, tol):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)
    assert err <= tol, err


# --- 1. explicit dense transition products --------------------------------

@pytest.mark.parametrize("dk,dv", [(5, 3), (4, 4), (3, 6)])
def test_dense_transition_product(dk, dv):
    """S_T = (prod M_t) S_0 + sum_i (prod_{j>i} M_j) beta_i k_i v_i^T with the
    dk x dk matrices M_t = (I - beta_t k_t k_t^T) Diag(alpha_t) formed densely.
    Non-square, non-symmetric S_0 so a transposed layout cannot pass."""
    T = 12
    q, k, v, g, beta, h0 = _rand(11 + dk, T, 1, dk, dv)
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    M = [(np.eye(dk) - beta[t, 0] * np.outer(k[t, 0], k[t, 0])) @ np.diag(np.exp(g[t, 0]))
         for t in range(T)]
    S0 = h0[0, 0]
    for t in range(T):
        # state after token t, built from products only (no running update)
        prod_all = np.eye(dk)
        for j in range(t + 1):
            prod_all = M[j] @ prod_all
        St = prod_all @ S0
        for i in range(t + 1):
            P = np.eye(dk)
            for j in range(i + 1, t + 1):
                P = M[j] @ P
            St = St + P @ (beta[i, 0] * np.outer(k[i, 0], v[i, 0]))
        _close(o[t, 0], St.T @ q[t, 0], 1e-12)
    _close(hN[0, 0], St, 1e-12)


# --- 2. special cases named on the pages -----------------------------------

def test_alpha_one_is_deltanet():
    """alpha = 1: the plain delta rule, written as 'predict, then store the
    difference' with a running S (Schlag et al. form)."""
    T, dk, dv = 20, 6, 5
    q, k, v, g, beta, h0 = _rand(3, T, 2, dk, dv)
    g[:] = 0.0
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    for h in range(2):
        S = h0[0, h].copy()
        for t in range(T):
            pred = S.T @ k[t, h]
            S = S + np.outer(k[t, h], beta[t, h] * (v[t, h] - pred))
            _close(o[t, h], S.T @ q[t, h], 1e-13)
        _close(hN[0, h], S, 1e-13)


def test_scalar_gate_is_gated_deltanet():
    """Head-uniform alpha: Gated DeltaNet, S = a (I - b k k^T) S + b k v^T; the
    scalar commutes with the projection."""
    T, dk, dv = 20, 7, 4
    q, k, v, g, beta, h0 = _rand(5, T, 1, dk, dv)
    gs = -np.log1p(np.exp(np.random.default_rng(9).standard_normal(T)))
    g[:] = gs[:, None, None]
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    S = h0[0, 0].copy()
    for t in range(T):
        a = np.exp(gs[t])
        S = a * (S - beta[t, 0] * np.outer(k[t, 0], k[t, 0] @ S)) + beta[t, 0] * np.outer(
            k[t, 0], v[t, 0])
        _close(o[t, 0], S.T @ q[t, 0], 1e-13)
    _close(hN[0, 0], S, 1e-13)


def test_beta_zero_is_pure_channel_decay():
    """beta = 0: S_t = Diag(exp(sum_{j<=t} g_j)) S_0 in closed form."""
    T, dk, dv = 30, 8, 4
    q, k, v, g, beta, h0 = _rand(7, T, 3, dk, dv)
    beta[:] = 0.0
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    cg = np.cumsum(g, axis=0)  # [T, H, dk]
    for h in range(3):
        for t in range(T):
            St = np.exp(cg[t, h])[:, None] * h0[0, h]
            _close(o[t, h], St.T @ q[t, h], 1e-13)
        _close(hN[0, h], np.exp(cg[-1, h])[:, None] * h0[0, h], 1e-13)


# --- 3. invariant: exact overwrite retrieval --------------------------------

def test_overwrite_retrieval_orthonormal_keys():
    """alpha = 1, beta = 1, orthonormal keys: after writing (k_i, v_i) the state
    returns v_i for k_i exactly, whatever it held before; rewriting a key
    returns the new value."""
    dk, dv, n = 16, 5, 10
    r = np.random.default_rng(1)
    Qm, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    keys = Qm[:, :n].T  # n orthonormal keys
    vals = r.standard_normal((n, dv))
    new_v = r.standard_normal(dv)
    T = n + 1 + n + 1
    k = np.zeros((T, 1, dk)); v = np.zeros((T, 1, dv)); q = np.zeros((T, 1, dk))
    k[:n, 0] = keys; v[:n, 0] = vals; q[:n, 0] = keys
    k[n, 0] = keys[0]; v[n, 0] = new_v; q[n, 0] = keys[0]       # rewrite key 0
    k[n + 1:, 0] = keys[0]; q[n + 1:2 * n + 1, 0] = keys       # read-only (beta = 0)
    beta = np.ones((T, 1)); beta[n + 1:] = 0.0
    g = np.zeros((T, 1, dk))
    h0 = r.standard_normal((1, 1, dk, dv))
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    for i in range(n):
        _close(o[i, 0], vals[i], 1e-13)           # read right after its write
    _close(o[n, 0], new_v, 1e-13)                  # overwrite in place
    for i in range(1, n):
        _close(o[n + 1 + i, 0], vals[i], 1e-13)   # other keys undisturbed
    _close(o[n + 1, 0], new_v, 1e-13)
    _close(hN[0, 0].T @ keys[0], new_v, 1e-13)


# --- 4. hand-worked example --------------------------------------------------

def test_hand_example_golden():
    ex = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    steps = ex["steps"]
    T = len(steps)
    q = np.array([s["q"] for s in steps])[:, None, :]
    k = np.array([s["k"] for s in steps])[:, None, :]
    v = np.array([s["v"] for s in steps])[:, None, :]
    g = np.log(np.array([s["alpha"] for s in steps]))[:, None, :]
    beta = np.array([s["beta"] for s in steps])[:, None]
    h0 = np.array(ex["S0"])[None, None]
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    for t in range(T):
        np.testing.assert_allclose(o[t, 0], steps[t]["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(hN[0, 0], steps[-1]["S"], rtol=0, atol=1e-12)
    # the same example one decode step at a time, with the state carried
    S = h0.copy()
    for t in range(T):
        ot, S = oracle.decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1],
                                   beta[t:t + 1], S)
        np.testing.assert_allclose(ot[0, 0], steps[t]["o"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(S[0, 0], steps[t]["S"], rtol=0, atol=1e-12)


# --- 5. composition ----------------------------------------------------------

def test_varlen_equals_separate_calls():
    lens = [5, 1, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = cu[-1]
    q, k, v, g, beta, h0 = _rand(21, T, 2, 6, 3, N=len(lens))
    o, hN = oracle.forward(q, k, v, g, beta, h0, cu_seqlens=cu)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        os_, hs = oracle.forward(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], h0[s:s + 1])
        np.testing.assert_array_equal(o[a:b], os_)
        np.testing.assert_array_equal(hN[s], hs[0])


def test_split_prefill_and_decode_compose():
    T = 23
    q, k, v, g, beta, h0 = _rand(31, T, 2, 5, 4)
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    o1, h1 = oracle.forward(q[:10], k[:10], v[:10], g[:10], beta[:10], h0)
    o2, h2 = oracle.forward(q[10:T - 1], k[10:T - 1], v[10:T - 1], g[10:T - 1], beta[10:T - 1],
                            h1)
    o3, h3 = oracle.decode_step(q[T - 1:], k[T - 1:], v[T - 1:], g[T - 1:], beta[T - 1:], h2)
    _close(np.concatenate([o1, o2, o3]), o, 1e-14)
    _close(h3, hN, 1e-14)


def test_batched_form_matches_cu_seqlens():
    B, T = 3, 7
    q, k, v, g, beta, h0 = _rand(41, B * T, 2, 4, 4, N=B)
    o_flat, h_flat = oracle.forward(q, k, v, g, beta, h0,
                                    cu_seqlens=np.arange(0, (B + 1) * T, T, dtype=np.int32))
    rs = lambda x: x.reshape(B, T, *x.shape[1:])
    o_b, h_b = oracle.forward(rs(q), rs(k), rs(v), rs(g), rs(beta), h0)
    np.testing.assert_array_equal(o_b.reshape(B * T, 2, 4), o_flat)
    np.testing.assert_array_equal(h_b, h_flat)


def test_zero_length_sequence_keeps_state():
    lens = [4, 0, 3]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g, beta, h0 = _rand(51, 7, 1, 4, 4, N=3)
    o, hN = oracle.forward(q, k, v, g, beta, h0, cu_seqlens=cu)
    np.testing.assert_array_equal(hN[1], h0[1])


def test_bad_cu_seqlens_rejected():
    q, k, v, g, beta, _ = _rand(1, 6, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, g, beta, cu_seqlens=np.array([0, 4, 3, 6], np.int32))
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, g, beta, cu_seqlens=np.array([0, 5], np.int32))


# --- 6. the chunkwise restatement against the recurrence ---------------------

@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunkwise_equals_recurrence(C):
    lens = [64, 37, 1, 100]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g, beta, h0 = _rand(61, cu[-1], 2, 8, 6, N=len(lens))
    o, hN = oracle.forward(q, k, v, g, beta, h0, cu_seqlens=cu)
    oc, hc = chunkwise.forward(q, k, v, g, beta, h0, cu_seqlens=cu, chunk=C)
    _close(oc, o, 1e-11)
    _close(hc, hN, 1e-11)


def test_chunkwise_strong_decay_stays_finite():
    """Strong decay (sum of g over a chunk near -300) must not overflow: the
    chunk form evaluates exp(G_r - G_i) directly."""
    T = 64
    q, k, v, g, beta, h0 = _rand(71, T, 1, 8, 8)
    g *= 6.0
    o, hN = oracle.forward(q, k, v, g, beta, h0)
    oc, hc = chunkwise.forward(q, k, v, g, beta, h0, chunk=64)
    assert np.isfinite(oc).all()
    _close(oc, o, 1e-11)
    _close(hc, hN, 1e-11)


def test_chunkwise_ut_transform_is_triangular_inverse():
    """T = (I + A)^{-1} is unit lower triangular and W, Ut satisfy the
    triangular systems (I + A) W = diag(b) (K * Gam), (I + A) Ut = diag(b) V."""
    q, k, v, g, beta, h0 = _rand(81, 16, 1, 6, 5)
    r = chunkwise.chunk_step(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], h0[0, 0])
    Tm, A = r["T"], r["A"]
    assert np.allclose(np.triu(Tm, 1), 0) and np.allclose(np.diag(Tm), 1)
    assert np.allclose(np.triu(A), 0)
    I = np.eye(16)
    _close((I + A) @ r["W"], beta[:, 0, None] * k[:, 0] * np.exp(r["G"]), 1e-13)
    _close((I + A) @ r["Ut"], beta[:, 0, None] * v[:, 0], 1e-13)
