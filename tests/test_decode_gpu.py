"""GPU parity of the fused decode step (kda_decode_step) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
import oracle
from gated_delta_rule_124_b200 import workloads as wl
from tests.helpers import ErrAccum, record, rel_err, tol_for

pytestmark = pytest.mark.gpu


def _run(case, steps, dev="cuda"):
    state = case.state0.to(dev).contiguous()
    outs = []
    for t in range(steps):
        s = case.steps[t % len(case.steps)]
        d = {k: v.to(dev).contiguous() for k, v in s.items()}
        o = kda.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], state)
        outs.append(o)
    torch.cuda.synchronize()
    return outs, state


def _oracle(case, steps, units=None):
    st = case.state0.numpy().astype(np.float64)
    outs = []
    for t in range(steps):
        s = case.steps[t % len(case.steps)]
        o, st = oracle.decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], st)
        outs.append(o)
    return outs, st


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (32, 32), (64, 32),
                                   (32, 128)])
def test_decode_small_shapes(dtype, dk, dv):
    case = wl.make_decode(7, N=3, H=5, dk=dk, dv=dv, dtype=dtype, sets=3)
    outs, state = _run(case, 5)
    r_outs, r_state = _oracle(case, 5)
    tol = tol_for(dtype)
    for o, ro in zip(outs, r_outs):
        assert rel_err(o, ro) <= tol
    assert rel_err(state, r_state) <= tol


def test_decode_full_config_all_steps():
    """The decode configuration at full extent: N=256 sequences x H=32 heads,
    128 x 128 fp32 states, all 1000 steps of the 8-set schedule; o of every
    step and the final state of every (sequence, head) against the fp64
    oracle.  The oracle replays each sequence's 1000 steps as one 1000-token
    recurrence (a decode step is one step of that recurrence), eight
    sequences at a time."""
    c = wl.DECODE_CONFIG
    case = wl.decode_config()
    steps, N, H, d = c["steps"], case.N, case.H, case.dk
    dev = "cuda"
    state = case.state0.to(dev).contiguous()
    dsets = [{k: v.to(dev).contiguous() for k, v in s.items()} for s in case.steps]
    o_all = torch.empty(steps, N, H, d, dtype=torch.bfloat16, device=dev)
    for t in range(steps):
        s = dsets[t % len(dsets)]
        kda.decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], state, o=o_all[t])
    torch.cuda.synchronize()
    acc_o, acc_s = ErrAccum(), ErrAccum()
    sched = [t % len(case.steps) for t in range(steps)]
    G = 8
    for n0 in range(0, N, G):
        n1 = min(N, n0 + G)
        seq = {k: torch.stack([case.steps[i][k][n0:n1] for i in sched], 1)
               for k in ("q", "k", "v", "g", "beta")}  # [n, steps, ...]
        flat = {k: v.reshape(-1, *v.shape[2:]) for k, v in seq.items()}
        cu = np.arange(0, (n1 - n0 + 1) * steps, steps, dtype=np.int32)
        ro, rs = oracle.forward(flat["q"], flat["k"], flat["v"], flat["g"], flat["beta"],
                                case.state0[n0:n1], cu_seqlens=cu)
        ro = ro.reshape(n1 - n0, steps, H, d).transpose(1, 0, 2, 3)
        acc_o.add(o_all[:, n0:n1], ro)
        acc_s.add(state[n0:n1], rs)
    eo = record(case.name, "o (all steps)", acc=acc_o)
    es = record(case.name, "state", acc=acc_s)
    assert eo <= tol_for(c["dtype"]), eo
    assert es <= tol_for(c["dtype"]), es


def test_decode_n_zero_is_noop():
    st = torch.randn(1, 2, 32, 32, device="cuda")
    before = st.clone()
    z = torch.empty(0, 2, 32, device="cuda")
    kda.kda_decode_step(z, z, z, z, torch.empty(0, 2, device="cuda"), st,
                        torch.empty(0, 2, 32, device="cuda"), 0, 2, 32, 32, "f32")
    torch.cuda.synchronize()
    assert torch.equal(st, before)


def test_decode_is_deterministic():
    case = wl.make_decode(9, N=4, H=8, dk=128, dv=128, dtype="bf16", sets=2)
    a, sa = _run(case, 3)
    b, sb = _run(case, 3)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert torch.equal(sa, sb)


def test_decode_matches_prefill_one_token():
    """A decode step equals a one-token prefill from the same state (shared
    state layout between the two paths)."""
    case = wl.make_decode(11, N=2, H=3, dk=64, dv=64, dtype="f32", sets=1)
    s = {k: v.cuda() for k, v in case.steps[0].items()}
    st = case.state0.cuda().clone()
    o_dec = kda.decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], st)
    cu = torch.arange(0, 3, dtype=torch.int32, device="cuda")
    o_pre, h_pre = kda.chunk_fwd(s["q"].reshape(2, 3, 64), s["k"].reshape(2, 3, 64),
                                 s["v"].reshape(2, 3, 64), s["g"].reshape(2, 3, 64),
                                 s["beta"].reshape(2, 3), case.state0.cuda(), cu_seqlens=cu,
                                 chunk=16)
    torch.cuda.synchronize()
    assert rel_err(o_dec, o_pre.reshape(2, 3, 64).double().cpu().numpy()) <= 1e-5
    assert rel_err(st, h_pre.double().cpu().numpy()) <= 1e-5
