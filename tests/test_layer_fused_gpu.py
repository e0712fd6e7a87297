"""GPU parity of the fused layer calls (the steps around the operator inside
the operator's kernels) against the fp64 composition of oracle/layer.py and
the KDA oracle, and against the unfused library calls."""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
import oracle
from oracle import layer
from tests.helpers import record, rel_err, tol_for

pytestmark = pytest.mark.gpu

EPS = 1e-6
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _decode_problem(seed, N, H, dk, dv, dtype, steps):
    g = torch.Generator().manual_seed(seed)
    dt = DT[dtype]
    xs = [[torch.randn(N, H, d, generator=g).to(dt) for d in (dk, dk, dv)] for _ in range(steps)]
    w = [torch.randn(H * d, 4, generator=g) * 0.5 for d in (dk, dk, dv)]
    conv = [(torch.randn(N, 3, H, d, generator=g) * 0.5).to(dt) for d in (dk, dk, dv)]
    gates = [-torch.nn.functional.softplus(torch.randn(N, H, dk, generator=g))
             for _ in range(steps)]
    betas = [torch.sigmoid(torch.randn(N, H, generator=g)) for _ in range(steps)]
    ogate = [torch.randn(N, H, dv, generator=g).to(dt) for _ in range(steps)]
    wn = torch.rand(dv, generator=g) + 0.5
    state = torch.randn(N, H, dk, dv, generator=g) * 0.02
    return xs, w, conv, gates, betas, ogate, wn, state


def _oracle_decode(xs, w, conv, gates, betas, ogate, wn, state):
    """fp64: per step, the 4-token window [c0, c1, c2, x] through the layer
    oracle's convolution (the last token's output), the KDA oracle's decode
    step, then RMSNorm and the output gate."""
    conv = [c.double().numpy().copy() for c in conv]  # [N, 3, H, d]
    st = state.double().numpy()
    ys = []
    for t, x in enumerate(xs):
        qkv = []
        for i in range(3):
            xi = x[i].double().numpy()  # [N, H, d]
            win = np.concatenate([conv[i], xi[:, None]], axis=1)  # [N, 4, H, d]
            N = win.shape[0]
            flat = win.reshape(N * 4, *win.shape[2:])
            cu = np.arange(0, 4 * N + 1, 4)
            y = layer.swish(layer.causal_conv4(flat, w[i], cu_seqlens=cu))
            y = y.reshape(N, 4, *win.shape[2:])[:, 3]
            qkv.append(layer.l2_normalize(y, EPS) if i < 2 else y)
            conv[i] = win[:, 1:]
        o, st = oracle.decode_step(qkv[0], qkv[1], qkv[2], gates[t], betas[t], st)
        ys.append(layer.output_norm_gate(o, ogate[t], wn, EPS))
    return ys, st, conv


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (32, 32)])
def test_layer_decode_matches_oracle(dtype, dk, dv):
    N, H, steps = 5, 3, 4
    xs, w, conv, gates, betas, ogate, wn, state = _decode_problem(31, N, H, dk, dv, dtype, steps)
    ry, rst, rconv = _oracle_decode(xs, w, conv, gates, betas, ogate, wn, state)
    d = lambda t: t.cuda().contiguous()  # noqa: E731
    wd, convd, std, wnd = [d(x) for x in w], [d(c) for c in conv], d(state), d(wn)
    tol = tol_for(dtype)
    for t in range(steps):
        y = torch.full_like(d(xs[t][2]), float("nan"))
        kda.kda_layer_decode_step(*[d(x) for x in xs[t]], *wd, *convd, d(gates[t]), d(betas[t]),
                                  std, d(ogate[t]), wnd, N, H, dk, dv, dtype, EPS, EPS, y)
        torch.cuda.synchronize()
        assert rel_err(y, ry[t]) <= tol, (t, rel_err(y, ry[t]))
    assert rel_err(std, rst) <= tol
    for c, rc in zip(convd, rconv):  # the states hold the last three raw inputs, exactly
        assert np.array_equal(c.double().cpu().numpy(), rc)


def test_layer_decode_full_size_matches_unfused_and_oracle():
    """N=256 sequences x H=32 heads, d = 128, bf16, 8 steps: the fused call
    against the fp64 composition (every output and the final state) and
    against the three unfused calls on the same inputs."""
    N, H, d, steps = 256, 32, 128, 8
    xs, w, conv, gates, betas, ogate, wn, state = _decode_problem(32, N, H, d, d, "bf16", steps)
    ry, rst, _ = _oracle_decode(xs, w, conv, gates, betas, ogate, wn, state)
    dv = lambda t: t.cuda().contiguous()  # noqa: E731
    wd = [dv(x) for x in w]
    conv_f, conv_u = [dv(c) for c in conv], [dv(c) for c in conv]
    st_f, st_u = dv(state), dv(state)
    wnd = dv(wn)
    ef, eu = [], []
    for t in range(steps):
        x = [dv(a) for a in xs[t]]
        g, b, og = dv(gates[t]), dv(betas[t]), dv(ogate[t])
        yf = torch.empty_like(x[2])
        kda.kda_layer_decode_step(*x, *wd, *conv_f, g, b, st_f, og, wnd, N, H, d, d, "bf16", EPS,
                                  EPS, yf)
        q, k, v = (torch.empty_like(a) for a in x)
        kda.kda_qkv_conv_norm_step(*x, *wd, *conv_u, N, H, d, d, "bf16", EPS, q, k, v)
        o = kda.decode_step(q, k, v, g, b, st_u)
        yu = torch.empty_like(o)
        kda.kda_output_norm_gate(o, og, wnd, N, H, d, "bf16", EPS, yu)
        torch.cuda.synchronize()
        ef.append(rel_err(yf, ry[t]))
        eu.append(rel_err(yf, yu.double().cpu().numpy()))
    record("layer decode step (fused): N=256 H=32 d=128 bf16", "y (step 8)", yf, ry[-1])
    assert max(ef) <= tol_for("bf16"), ef
    assert max(eu) <= tol_for("bf16"), eu
    assert rel_err(st_f, rst) <= tol_for("bf16")
    for a, b in zip(conv_f, conv_u):
        assert torch.equal(a, b)


# ------------------------------------------------------------------ prefill

def _prefill_problem(seed, lens, H, dk, dv, dtype):
    g = torch.Generator().manual_seed(seed)
    dt = DT[dtype]
    total = sum(lens)
    x = [torch.randn(total, H, d, generator=g).to(dt) for d in (dk, dk, dv)]
    w = [torch.randn(H * d, 4, generator=g) * 0.5 for d in (dk, dk, dv)]
    gk = -torch.nn.functional.softplus(torch.randn(total, H, dk, generator=g))
    beta = torch.sigmoid(torch.randn(total, H, generator=g))
    ogate = torch.randn(total, H, dv, generator=g).to(dt)
    wn = torch.rand(dv, generator=g) + 0.5
    h0 = torch.randn(len(lens), H, dk, dv, generator=g) * 0.02
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return x, w, gk, beta, ogate, wn, h0, cu


def _oracle_prefill_layer(x, w, gk, beta, ogate, wn, h0, cu):
    q, k, v = layer.qkv_conv_norm(*x, *w, cu_seqlens=cu, eps=EPS)
    o, hN = oracle.forward(q, k, v, gk, beta, h0, cu_seqlens=cu)
    return layer.output_norm_gate(o, ogate, wn, EPS), hN


def _run_prefill_layer(x, w, gk, beta, ogate, wn, h0, cu, H, dk, dv, C, dtype):
    d = lambda t: t.cuda().contiguous()  # noqa: E731
    total, N = int(cu[-1]), len(cu) - 1
    cud = torch.tensor(cu, dtype=torch.int32, device="cuda")
    y = torch.full_like(d(x[2]), float("nan"))
    hN = torch.full((N, H, dk, dv), float("nan"), device="cuda")
    ws = torch.empty(kda.kda_layer_chunk_fwd_workspace_size(total, N, H, dk, dv, C, dtype),
                     dtype=torch.uint8, device="cuda")
    kda.kda_layer_chunk_fwd(*[d(a) for a in x], *[d(a) for a in w], d(gk), d(beta), d(h0), cud,
                            1, total, N, H, dk, dv, C, dtype, d(ogate), d(wn), EPS, EPS, y, hN, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    return y, hN


@pytest.mark.parametrize("dtype,dk,dv,C", [("bf16", 128, 128, 64), ("f32", 64, 32, 32),
                                           ("bf16", 64, 64, 16)])
def test_layer_prefill_matches_oracle(dtype, dk, dv, C):
    """Packed sequences with a 1-token one, one shorter than a chunk, and
    several chunks (the rows before a chunk come from the previous chunk)."""
    lens = [C * 3 + 5, 1, C - 3, 2 * C]
    H = 3
    args = _prefill_problem(41, lens, H, dk, dv, dtype)
    ry, rh = _oracle_prefill_layer(*args)
    y, hN = _run_prefill_layer(*args, H, dk, dv, C, dtype)
    tol = tol_for(dtype)
    assert rel_err(y, ry) <= tol, rel_err(y, ry)
    assert rel_err(hN, rh) <= tol, rel_err(hN, rh)


def test_layer_prefill_full_size_matches_unfused_and_oracle():
    """B=2 x T=2048 tokens, H=32, d=128, bf16: the fused call against the fp64
    composition (every output and final state) and against the three unfused
    library calls on the same inputs."""
    lens, H, d = [2048, 2048], 32, 128
    x, w, gk, beta, ogate, wn, h0, cu = _prefill_problem(42, lens, H, d, d, "bf16")
    ry, rh = _oracle_prefill_layer(x, w, gk, beta, ogate, wn, h0, cu)
    y, hN = _run_prefill_layer(x, w, gk, beta, ogate, wn, h0, cu, H, d, d, 64, "bf16")
    eo, eh = record("layer prefill (fused): B=2 T=2048 H=32 d=128 bf16", "y", y, ry), \
        record("layer prefill (fused): B=2 T=2048 H=32 d=128 bf16", "final_state", hN, rh)
    assert eo <= tol_for("bf16") and eh <= tol_for("bf16"), (eo, eh)
    # the unfused path
    dv_ = lambda t: t.cuda().contiguous()  # noqa: E731
    cud = torch.tensor(cu, dtype=torch.int32, device="cuda")
    xs = [dv_(a) for a in x]
    q, k, v = (torch.empty_like(a) for a in xs)
    kda.kda_qkv_conv_norm(*xs, *[dv_(a) for a in w], cud, 1, 4096, 2, H, d, d, "bf16", EPS,
                          q, k, v)
    o, hu = kda.chunk_fwd(q, k, v, dv_(gk), dv_(beta), dv_(h0), cu_seqlens=cud, chunk=64)
    yu = torch.empty_like(o)
    kda.kda_output_norm_gate(o, dv_(ogate), dv_(wn), 4096, H, d, "bf16", EPS, yu)
    torch.cuda.synchronize()
    assert rel_err(y, yu.double().cpu().numpy()) <= tol_for("bf16")
    assert rel_err(hN, hu.double().cpu().numpy()) <= tol_for("bf16")
