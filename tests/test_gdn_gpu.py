"""Gated DeltaNet (one gate value per (token, head)) through kda_gdn_chunk_fwd
and kda_gdn_decode_step, against the fp64 oracle run on the gate spread over
the key channels (the head-uniform gate is the special case of KDA's
per-channel gate), on both plans."""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
import oracle
from gated_delta_rule_124_b200 import workloads as wl
from tests.helpers import rel_err, tol_for

pytestmark = pytest.mark.gpu


def _head_gate(case, seed, mu=0.0, scale=1.0):
    """A head-uniform log-gate [total, H] (−softplus of a normal, like the
    per-channel one), and the same gate spread over dk."""
    g = torch.Generator().manual_seed(seed)
    gh = -torch.nn.functional.softplus(torch.randn(case.total, case.H, generator=g) + mu) * scale
    return gh, gh[:, :, None].expand(case.total, case.H, case.dk).contiguous()


def _run(case, gh):
    c = case.to("cuda")
    B, T = (1, c.total) if c.cu_seqlens is not None else (c.B, c.T)
    ws = torch.empty(kda.kda_gdn_chunk_fwd_workspace_size(c.total, c.N, c.H, c.dk, c.dv,
                                                          c.chunk, c.dtype),
                     dtype=torch.uint8, device="cuda")
    o = torch.full_like(c.v, float("nan"))
    hN = torch.full((c.N, c.H, c.dk, c.dv), float("nan"), device="cuda")
    kda.kda_gdn_chunk_fwd(c.q, c.k, c.v, gh.cuda(), c.beta, c.initial_state, c.cu_seqlens, B, T,
                          c.N, c.H, c.dk, c.dv, c.chunk, c.dtype, o, hN, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    return o, hN


def _check(case, gh, gfull):
    o, hN = _run(case, gh)
    cu = case.cu_host() if case.cu_seqlens is not None else None
    ro, rh = oracle.forward(case.q, case.k, case.v, gfull, case.beta, case.initial_state, cu)
    tol = tol_for(case.dtype)
    assert rel_err(o, ro) <= tol and rel_err(hN, rh) <= tol, (rel_err(o, ro), rel_err(hN, rh))
    return o, hN


@pytest.mark.parametrize("d,C", [(128, 64), (64, 32)])
def test_gdn_prefill_bf16(d, C):
    """d = 128, chunk 64: the split tensor-core plan with the gate read per
    (token, head); d = 64: the gate spread over the channels, CUDA-core plan."""
    case = wl.make_prefill(401, [300, 77, 1, 128], H=4, dk=d, dv=d, chunk=C,
                           dtype="bf16", varlen=True)
    gh, gfull = _head_gate(case, 1)
    _check(case, gh, gfull)


def test_gdn_prefill_fp32_small():
    case = wl.make_prefill(402, [100, 37], H=2, dk=64, dv=32, chunk=16, dtype="f32",
                           varlen=True)
    gh, gfull = _head_gate(case, 2)
    _check(case, gh, gfull)


def test_gdn_strong_decay_takes_the_exact_path():
    # per-token log-decay around -6: a chunk's range far beyond the factorised
    # form's headroom, so every chunk is evaluated exactly
    case = wl.make_prefill(403, [200], H=2, dk=128, dv=128, chunk=64, dtype="bf16")
    gh, gfull = _head_gate(case, 3, mu=6.0)
    _check(case, gh, gfull)


def test_deltanet_is_gdn_with_zero_gate():
    case = wl.make_prefill(404, [190], H=2, dk=128, dv=128, chunk=64, dtype="bf16")
    gh = torch.zeros(case.total, case.H)
    _check(case, gh, torch.zeros(case.total, case.H, case.dk))


def test_gdn_long_sequence_takes_the_co_scheduled_plan():
    """One 16384-token sequence over 16 heads: few long chains, so the plan
    rule picks the co-scheduled launch (intra units of the head-gate variant
    beside the chain units); against the oracle on the spread gate."""
    case = wl.make_prefill(406, [16384], H=16, dk=128, dv=128, chunk=64, dtype="bf16")
    assert kda.PLAN_NAMES[kda.kda_chunk_fwd_plan(case.total, case.N, case.H, 128, 128, 64,
                                                 "bf16")] == "overlap"
    gh, gfull = _head_gate(case, 6)
    _check(case, gh, gfull)


def test_gdn_agrees_with_kda_on_a_spread_gate():
    case = wl.make_prefill(405, [256, 130], H=3, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    gh, gfull = _head_gate(case, 4)
    o1, h1 = _run(case, gh)
    c = case.to("cuda")
    o2, h2 = kda.chunk_fwd(c.q, c.k, c.v, gfull.cuda(), c.beta, c.initial_state, c.cu_seqlens)
    assert rel_err(o1, o2.double().cpu().numpy()) <= 1e-2
    assert rel_err(h1, h2.double().cpu().numpy()) <= 2e-3


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gdn_decode(dtype):
    g = torch.Generator().manual_seed(5)
    N, H, d = 9, 3, 128
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.nn.functional.normalize(torch.randn(N, H, d, generator=g), dim=-1).to(tdt)
    k = torch.nn.functional.normalize(torch.randn(N, H, d, generator=g), dim=-1).to(tdt)
    v = torch.randn(N, H, d, generator=g).to(tdt)
    gh = -torch.nn.functional.softplus(torch.randn(N, H, generator=g))
    beta = torch.sigmoid(torch.randn(N, H, generator=g))
    s0 = torch.randn(N, H, d, d, generator=g) * 0.02
    st = s0.clone().cuda()
    o = torch.empty(N, H, d, dtype=tdt, device="cuda")
    kda.kda_gdn_decode_step(q.cuda(), k.cuda(), v.cuda(), gh.cuda(), beta.cuda(), st, o, N, H,
                            d, d, dtype)
    torch.cuda.synchronize()
    ro, rs = oracle.decode_step(q, k, v, gh[:, :, None].expand(N, H, d).contiguous(), beta, s0)
    tol = 2e-2 if dtype == "bf16" else 1e-4
    assert rel_err(o, ro) <= tol and rel_err(st, rs) <= tol
