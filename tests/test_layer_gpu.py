"""GPU parity of the steps around the operator (kda_qkv_conv_norm,
kda_output_norm_gate) against the fp64 oracle in oracle/layer.py."""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
from oracle import layer
from tests.helpers import rel_err

pytestmark = pytest.mark.gpu

EPS = 1e-6
TOL = {"bf16": 1e-2, "f32": 1e-5}
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _inputs(seed, total, H, dk, dv, dtype):
    g = torch.Generator().manual_seed(seed)
    x = [torch.randn(total, H, d, generator=g).to(DT[dtype]) for d in (dk, dk, dv)]
    w = [(torch.randn(H * d, 4, generator=g) * 0.5) for d in (dk, dk, dv)]
    return x, w


def _run_conv(x, w, cu, B, T, N, H, dk, dv, dtype):
    dev = [t.cuda() for t in x]
    wd = [t.cuda() for t in w]
    out = [torch.full_like(t, float("nan")) for t in dev]
    cud = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    kda.kda_qkv_conv_norm(*dev, *wd, cud, B, T, N, H, dk, dv, dtype, EPS, *out)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 128)])
def test_conv_norm_matches_oracle(dtype, dk, dv):
    B, T, H = 2, 77, 3
    x, w = _inputs(11, B * T, H, dk, dv, dtype)
    q, k, v = _run_conv(x, w, None, B, T, B, H, dk, dv, dtype)
    cu = [0, T, 2 * T]
    rq, rk, rv = layer.qkv_conv_norm(*x, *w, cu_seqlens=cu, eps=EPS)
    for got, ref in ((q, rq), (k, rk), (v, rv)):
        assert rel_err(got, ref) <= TOL[dtype]


def test_conv_norm_packed_sequences():
    lens = [5, 1, 0, 130, 2]
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    total, H = cu[-1], 2
    x, w = _inputs(12, total, H, 128, 128, "bf16")
    q, k, v = _run_conv(x, w, cu, 1, total, len(lens), H, 128, 128, "bf16")
    rq, rk, rv = layer.qkv_conv_norm(*x, *w, cu_seqlens=cu, eps=EPS)
    for got, ref in ((q, rq), (k, rk), (v, rv)):
        assert rel_err(got, ref) <= TOL["bf16"]
    # unit length per (token, head) for q and k
    nq = torch.linalg.vector_norm(q.float(), dim=-1)
    assert torch.allclose(nq, torch.ones_like(nq), atol=1e-2)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dv", [128, 64, 32])
def test_output_norm_gate_matches_oracle(dtype, dv):
    g = torch.Generator().manual_seed(13)
    total, H = 301, 4
    o = (torch.randn(total, H, dv, generator=g) * 3).to(DT[dtype])
    gate = torch.randn(total, H, dv, generator=g).to(DT[dtype])
    w = torch.randn(dv, generator=g)
    y = torch.full_like(o, float("nan")).cuda()
    kda.kda_output_norm_gate(o.cuda(), gate.cuda(), w.cuda(), total, H, dv, dtype, EPS, y)
    torch.cuda.synchronize()
    assert rel_err(y, layer.output_norm_gate(o, gate, w, eps=EPS)) <= TOL[dtype]


def test_output_norm_gate_in_place():
    g = torch.Generator().manual_seed(14)
    o = torch.randn(64, 2, 128, generator=g).to(torch.bfloat16)
    gate = torch.randn(64, 2, 128, generator=g).to(torch.bfloat16)
    w = torch.ones(128)
    od = o.cuda()
    kda.kda_output_norm_gate(od, gate.cuda(), w.cuda(), 64, 2, 128, "bf16", EPS, od)
    torch.cuda.synchronize()
    assert rel_err(od, layer.output_norm_gate(o, gate, w, eps=EPS)) <= TOL["bf16"]


def test_layer_steps_around_the_operator():
    """conv/Swish/L2-norm -> kda_chunk_fwd -> RMSNorm/gate, against the same
    chain of oracles (the operator's oracle is the fp64 recurrence)."""
    import oracle
    from gated_delta_rule_124_b200 import workloads as wl
    B, T, H, d = 1, 200, 2, 128
    x, w = _inputs(15, B * T, H, d, d, "bf16")
    q, k, v = _run_conv(x, w, None, B, T, B, H, d, d, "bf16")
    case = wl.make_prefill(16, [T], H=H, dk=d, dv=d, chunk=64, dtype="bf16")
    g_, beta = case.g.cuda(), case.beta.cuda()
    o, _ = kda.chunk_fwd(q.view(B, T, H, d), k.view(B, T, H, d), v.view(B, T, H, d),
                         g_.view(B, T, H, d), beta.view(B, T, H), output_final_state=False)
    gate = torch.randn(B * T, H, d).to(torch.bfloat16)
    wn = torch.rand(d) + 0.5
    y = torch.empty_like(o).view(B * T, H, d)
    kda.kda_output_norm_gate(o.view(B * T, H, d), gate.cuda(), wn.cuda(), B * T, H, d, "bf16",
                             EPS, y)
    torch.cuda.synchronize()
    # reference: oracle steps on the GPU's bf16 q, k, v (the operator's input
    # rounding is not the layer's error), then the recurrence, then the gate
    ro, _ = oracle.forward(q.cpu(), k.cpu(), v.cpu(), case.g, case.beta,
                           torch.zeros(1, H, d, d), None)
    ry = layer.output_norm_gate(ro, gate, wn, eps=EPS)
    assert rel_err(y, ry) <= 2e-2


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32)])
def test_conv_step_continues_a_prefill(dtype, dk, dv):
    """Decode-time convolution: a prefill over the first 5 tokens of each of 3
    sequences, the state taken from their last three input rows, then two
    steps; and steps from a zero state from the first token.  Both against the
    prefill convolution of all 7 tokens and the oracle."""
    B, T, H, T0 = 3, 7, 2, 5
    x, w = _inputs(31, B * T, H, dk, dv, dtype)
    full = _run_conv(x, w, None, B, T, B, H, dk, dv, dtype)
    ref = layer.qkv_conv_norm(*x, *w, cu_seqlens=np.arange(B + 1) * T, eps=EPS)
    wd = [t.cuda() for t in w]
    xs = [t.cuda().reshape(B, T, H, -1) for t in x]
    for start in (0, T0):
        # state: the last three inputs before `start` (zeros before the sequence)
        st = []
        for xt in xs:
            s = torch.zeros(B, 3, H, xt.shape[-1], dtype=xt.dtype, device="cuda")
            for i in range(3):
                t = start - 3 + i
                if t >= 0:
                    s[:, i] = xt[:, t]
            st.append(s)
        for t in range(start, T):
            xt = [a[:, t].contiguous() for a in xs]
            out = [torch.full_like(a, float("nan")) for a in xt]
            kda.kda_qkv_conv_norm_step(*xt, *wd, *st, B, H, dk, dv, dtype, EPS, *out)
            torch.cuda.synchronize()
            for j in range(3):
                f = full[j].reshape(B, T, H, -1)[:, t]
                r = ref[j].reshape(B, T, H, -1)[:, t]
                assert rel_err(out[j], r) <= TOL[dtype], (start, t, j)
                same = 1e-6 if dtype == "f32" else TOL[dtype]  # bf16: one rounding apart
                assert rel_err(out[j], f.float().cpu().numpy()) <= same, (start, t, j)
