"""GPU parity of kda_chunk_bwd against the fp64 autograd oracle
(oracle/backward.py, pinned by finite differences)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
from gated_delta_rule_124_b200 import workloads as wl
from oracle import backward as bwd
from tests.helpers import record, rel_err

pytestmark = pytest.mark.gpu


def _run(case, do, dhT):
    c = case.to("cuda")
    packed = c.cu_seqlens is not None
    B, T = (1, c.total) if packed else (c.B, c.T)
    f32 = dict(dtype=torch.float32, device="cuda")
    dq = torch.full((c.total, c.H, c.dk), float("nan"), **f32)
    dk = torch.full_like(dq, float("nan"))
    dg = torch.full_like(dq, float("nan"))
    dv = torch.full((c.total, c.H, c.dv), float("nan"), **f32)
    db = torch.full((c.total, c.H), float("nan"), **f32)
    dh0 = torch.full((c.N, c.H, c.dk, c.dv), float("nan"), **f32)
    ws = torch.empty(kda.kda_chunk_bwd_workspace_size(c.total, c.N, c.H, c.dk, c.dv),
                     dtype=torch.uint8, device="cuda")
    kda.kda_chunk_bwd(c.q, c.k, c.v, c.g, c.beta, c.initial_state, do.cuda(),
                      None if dhT is None else dhT.cuda(), c.cu_seqlens, B, T, c.N, c.H, c.dk,
                      c.dv, c.dtype, dq, dk, dv, dg, db, dh0, ws)
    torch.cuda.synchronize()
    return dq, dk, dv, dg, db, dh0


CASES = {
    "bf16_d128_varlen": lambda: wl.make_prefill(501, [40, 17, 0, 70], H=2, dk=128, dv=128,
                                                chunk=64, dtype="bf16", varlen=True),
    "f32_d64_dv32": lambda: wl.make_prefill(502, [33, 9], H=3, dk=64, dv=32, chunk=16,
                                            dtype="f32", varlen=True),
    "bf16_batched_d32": lambda: wl.make_prefill(503, [25, 25], H=2, dk=32, dv=64, chunk=16,
                                                dtype="bf16"),
    # several 64-token chunks per sequence, ragged tails, an exact multiple
    "bf16_d128_multichunk": lambda: wl.make_prefill(504, [150, 64, 129], H=2, dk=128, dv=128,
                                                    chunk=64, dtype="bf16", varlen=True),
    "f32_d128_dv64_batched": lambda: wl.make_prefill(505, [200, 200], H=1, dk=128, dv=64,
                                                     chunk=64, dtype="f32"),
    # fp32 inputs through the tensor-core kernels (dk = dv = 128)
    "f32_d128_varlen": lambda: wl.make_prefill(507, [90, 0, 130], H=2, dk=128, dv=128,
                                               chunk=64, dtype="f32", varlen=True),
}


def _strong_decay():
    """Gates twenty times stronger: the states forget within a few tokens and
    exp(G) of a whole chunk underflows, while every pairwise factor stays
    finite."""
    case = wl.make_prefill(506, [130, 70], H=2, dk=64, dv=64, chunk=64, dtype="f32",
                           varlen=True)
    case.g = case.g * 20.0
    return case


CASES["f32_d64_strong_decay"] = _strong_decay


def _mixed_decay_d128():
    """dk = dv = 128 with the second sequence's gates twenty times stronger:
    its chunks exceed the exponent reference's range and are recomputed by
    the exact kernels, the first sequence's chunks are not — both kinds in
    one call."""
    case = wl.make_prefill(511, [130, 70], H=2, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    case.g[130:] = case.g[130:] * 20.0
    return case


CASES["bf16_d128_mixed_decay"] = _mixed_decay_d128


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("with_dhT", [True, False])
def test_backward_matches_autograd(name, with_dhT):
    case = CASES[name]()
    g = torch.Generator().manual_seed(7)
    dt = torch.bfloat16 if case.dtype == "bf16" else torch.float32
    do = torch.randn(case.total, case.H, case.dv, generator=g).to(dt)
    dhT = torch.randn(case.N, case.H, case.dk, case.dv, generator=g) if with_dhT else None
    got = _run(case, do, dhT)
    cu = case.cu_host() if case.cu_seqlens is not None else np.arange(case.N + 1) * case.T
    ref = bwd.backward(case.q, case.k, case.v, case.g, case.beta, case.initial_state, do,
                       dhT, cu)
    for name_, x, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref):
        e = record(f"backward {name} {'with' if with_dhT else 'no'} dS_T", name_, x, r)
        assert e <= 1e-3, (name_, e)


@pytest.mark.parametrize("unit", [(0, 0), (1, 31)])
def test_backward_bench_workload_sampled_heads(unit):
    """The bench's prefill workload (B=2, T=2048, H=32, d=128, bf16) in the
    launch configuration the bench times; the oracle's gradients of one
    (sequence, head) at a time -- heads are independent, so the slice is an
    exact reference for that head's outputs."""
    case = wl.prefill_config(1)
    s, h = unit
    g = torch.Generator().manual_seed(11)
    do = torch.randn(case.total, case.H, case.dv, generator=g).to(torch.bfloat16)
    dhT = torch.randn(case.N, case.H, case.dk, case.dv, generator=g)
    got = _run(case, do, dhT)
    rows = slice(s * case.T, (s + 1) * case.T)
    one = lambda x: x[rows, h:h + 1]
    h0 = case.initial_state[s:s + 1, h:h + 1] if case.initial_state is not None else None
    if h0 is None:
        h0 = torch.zeros(1, 1, case.dk, case.dv)
    ref = bwd.backward(one(case.q), one(case.k), one(case.v), one(case.g),
                       case.beta[rows, h:h + 1], h0, one(do), dhT[s:s + 1, h:h + 1],
                       np.array([0, case.T]))
    sel = (one(got[0]), one(got[1]), one(got[2]), one(got[3]), got[4][rows, h:h + 1],
           got[5][s:s + 1, h:h + 1])
    for name_, x, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), sel, ref):
        e = record(f"backward B=2 T=2048 H=32 d=128 bf16 (seq {s}, head {h})", name_, x, r)
        assert e <= 1e-3, (name_, e)


def test_backward_bad_cu_seqlens_reported_on_device():
    """Invalid device cu_seqlens: the chunk table flags them, every later kernel
    returns before reading them, and the status word says so; a good call on
    the same workspace clears it."""
    case = wl.make_prefill(508, [40, 40], H=1, dk=32, dv=32, chunk=64, dtype="f32", varlen=True)
    c = case.to("cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    outs = [torch.zeros(80, 1, 32, **f32) for _ in range(4)]
    db, dh0 = torch.zeros(80, 1, **f32), torch.zeros(2, 1, 32, 32, **f32)
    do = torch.randn(80, 1, 32, device="cuda")
    ws = torch.empty(kda.kda_chunk_bwd_workspace_size(80, 2, 1, 32, 32), dtype=torch.uint8,
                     device="cuda")
    call = lambda cu: kda.kda_chunk_bwd(c.q, c.k, c.v, c.g, c.beta, None, do, None, cu, 1, 80, 2,
                                        1, 32, 32, "f32", outs[0], outs[1], outs[2], outs[3],
                                        db, dh0, ws)
    call(torch.tensor([0, 50, 40], dtype=torch.int32, device="cuda"))  # not monotone
    assert kda.kda_get_device_status(ws) == kda.KDA_ERR_BAD_SEQLENS
    call(torch.tensor([0, 30, 70], dtype=torch.int32, device="cuda"))  # wrong total
    assert kda.kda_get_device_status(ws) == kda.KDA_ERR_BAD_SEQLENS
    call(c.cu_seqlens)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK


@pytest.mark.parametrize("with_dhT", [True, False])
def test_gdn_backward_head_gate(with_dhT):
    """Gated DeltaNet: one gate value per (token, head).  The oracle runs on the
    gate spread over the dk channels; the gate's gradient is the sum of the
    per-channel ones (the chain rule of the spread)."""
    case = wl.make_prefill(509, [70, 0, 45], H=2, dk=64, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    gen = torch.Generator().manual_seed(13)
    gh = -torch.nn.functional.softplus(torch.randn(case.total, case.H, generator=gen))
    do = torch.randn(case.total, case.H, case.dv, generator=gen).to(torch.bfloat16)
    dhT = torch.randn(case.N, case.H, case.dk, case.dv, generator=gen) if with_dhT else None
    c = case.to("cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    dq = torch.full((c.total, c.H, c.dk), float("nan"), **f32)
    dk, dv = torch.full_like(dq, float("nan")), torch.full((c.total, c.H, c.dv), float("nan"), **f32)
    dg = torch.full((c.total, c.H), float("nan"), **f32)
    db = torch.full((c.total, c.H), float("nan"), **f32)
    dh0 = torch.full((c.N, c.H, c.dk, c.dv), float("nan"), **f32)
    ws = torch.empty(kda.kda_gdn_chunk_bwd_workspace_size(c.total, c.N, c.H, c.dk, c.dv),
                     dtype=torch.uint8, device="cuda")
    kda.kda_gdn_chunk_bwd(c.q, c.k, c.v, gh.cuda(), c.beta, c.initial_state, do.cuda(),
                          None if dhT is None else dhT.cuda(), c.cu_seqlens, 1, c.total, c.N,
                          c.H, c.dk, c.dv, "bf16", dq, dk, dv, dg, db, dh0, ws)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    g_full = gh[:, :, None].expand(-1, -1, case.dk).contiguous()
    ref = bwd.backward(case.q, case.k, case.v, g_full, case.beta, case.initial_state, do, dhT,
                       case.cu_host())
    ref_dg = ref[3].sum(axis=2)
    for name_, x, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"),
                           (dq, dk, dv, dg, db, dh0),
                           (ref[0], ref[1], ref[2], ref_dg, ref[4], ref[5])):
        assert rel_err(x, r) <= 1e-3, (name_, rel_err(x, r))


@pytest.mark.parametrize("head_gate", [False, True])
def test_autograd_function_matches_oracle(head_gate):
    """chunk_kda (forward + backward through autograd) against the oracle's
    gradients: q, k, v gradients come back in bf16 (their inputs' dtype), the
    rest in fp32."""
    case = wl.make_prefill(510, [90, 40], H=2, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    gen = torch.Generator().manual_seed(17)
    g_in = (-torch.nn.functional.softplus(torch.randn(case.total, case.H, generator=gen))
            if head_gate else case.g)
    do = torch.randn(case.total, case.H, case.dv, generator=gen).to(torch.bfloat16)
    dhT = torch.randn(case.N, case.H, case.dk, case.dv, generator=gen)
    leaves = [x.cuda().requires_grad_(True)
              for x in (case.q, case.k, case.v, g_in, case.beta, case.initial_state)]
    o, hN = kda.chunk_kda(*leaves, cu_seqlens=case.cu_seqlens.cuda(), head_gate=head_gate)
    loss = (o.float() * do.cuda().float()).sum() + (hN * dhT.cuda()).sum()
    loss.backward()
    g_full = g_in[:, :, None].expand(-1, -1, case.dk).contiguous() if head_gate else g_in
    ref = list(bwd.backward(case.q, case.k, case.v, g_full, case.beta, case.initial_state, do,
                            dhT, case.cu_host()))
    if head_gate:
        ref[3] = ref[3].sum(axis=2)
    tol = (1e-2, 1e-2, 1e-2, 1e-3, 1e-3, 1e-3)  # bf16-rounded q, k, v gradients
    for name_, x, r, t in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), leaves, ref, tol):
        assert x.grad is not None and x.grad.dtype == x.dtype, name_
        assert rel_err(x.grad, r) <= t, (name_, rel_err(x.grad, r))


def test_backward_no_tokens():
    """No tokens at all: the state gradient passes through unchanged
    (dS_0 = dS_T), for one sequence and for several empty ones."""
    for N in (1, 3):
        cu = torch.zeros(N + 1, dtype=torch.int32, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        e = torch.zeros(64, **f32)  # token arrays: valid pointers, nothing read or written
        dhT = torch.randn(N, 2, 32, 32, **f32)
        dh0 = torch.full_like(dhT, float("nan"))
        ws = torch.empty(max(kda.kda_chunk_bwd_workspace_size(0, N, 2, 32, 32), 256),
                         dtype=torch.uint8, device="cuda")
        kda.kda_chunk_bwd(e, e, e, e, e, None, e, dhT, cu, 1, 0, N, 2, 32, 32, "f32", e, e, e,
                          e, e, dh0, ws)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status(ws) == kda.KDA_OK
        assert torch.equal(dh0, dhT)
