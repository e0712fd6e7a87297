"""kda_chunk_fwd_noalloc: prefill for callers that may not allocate device memory.

Some callers are handed only their inputs and outputs -- an operator inside an
engine whose memory planner owns the whole device, or a serving loop that
reserved nearly all HBM up front -- and cannot pass a workspace.  This entry
point uses a static scratch array inside the library instead.  The GPU test
calls it twice in a row, through the C ABI, on two different problems (so the
second call runs on scratch the first one left behind) and compares each
result with kda_chunk_fwd's and with the fp64 oracle's, and reads the device's free memory around the
calls: the static array is committed by the first call (lazy module loading)
or before it (eager loading), never by a later one.  This file is collected
last on purpose.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
from gated_delta_rule_124_b200 import workloads as wl
from tests.helpers import oracle_prefill, record, rel_err, tol_for


def _problem(seed, lens, H, d, C, dtype):
    return wl.make_prefill(seed, lens, H=H, dk=d, dv=d, chunk=C, dtype=dtype, varlen=True)


def _with_workspace(c):
    ws = kda.alloc_workspace(c.total, c.N, c.H, c.dk, c.dv, c.chunk, c.dtype)
    o = torch.empty_like(c.v)
    hN = torch.empty(c.N, c.H, c.dk, c.dv, device="cuda")
    kda.kda_chunk_fwd(c.q, c.k, c.v, c.g, c.beta, c.initial_state, c.cu_seqlens, 1, c.total,
                      c.N, c.H, c.dk, c.dv, c.chunk, c.dtype, o, hN, ws)
    return o, hN


def _no_alloc(c):
    o = torch.full_like(c.v, float("nan"))
    hN = torch.full((c.N, c.H, c.dk, c.dv), float("nan"), device="cuda")
    kda.kda_chunk_fwd_noalloc(c.q, c.k, c.v, c.g, c.beta, c.initial_state, c.cu_seqlens, 1,
                              c.total, c.N, c.H, c.dk, c.dv, c.chunk, c.dtype, o, hN)
    return o, hN


@pytest.mark.gpu
def test_no_alloc_commits_its_scratch_once():
    """Free device memory around the calls (torch allocates nothing in
    between): the first call takes either the whole static array (lazy module
    loading: the driver loads the array's module on that call) or nothing
    (eager loading, or an earlier call already did); a repeated call takes
    nothing."""
    c = _problem(503, [130, 7], H=2, d=64, C=32, dtype="f32").to("cuda")
    _with_workspace(c)  # loads the CUDA-core kernels this problem runs
    o = torch.empty_like(c.v)
    hN = torch.empty(c.N, c.H, c.dk, c.dv, device="cuda")
    torch.cuda.synchronize()
    mib = 1 << 20
    free0 = torch.cuda.mem_get_info()[0]
    for i in range(2):
        kda.kda_chunk_fwd_noalloc(c.q, c.k, c.v, c.g, c.beta, c.initial_state, c.cu_seqlens, 1,
                                  c.total, c.N, c.H, c.dk, c.dv, c.chunk, c.dtype, o, hN)
        torch.cuda.synchronize()
        if i == 0:
            free1 = torch.cuda.mem_get_info()[0]
    free2 = torch.cuda.mem_get_info()[0]
    first = free0 - free1
    assert abs(first) <= 4 * mib or \
        abs(first - kda.KDA_NOALLOC_SCRATCH_BYTES) <= 4 * mib, first / mib
    assert free1 - free2 == 0, (free1 - free2) / mib


@pytest.mark.gpu
def test_no_alloc_matches_workspace_entry_point_and_oracle_twice():
    """Each result against kda_chunk_fwd's and, directly, against the fp64
    oracle on the same inputs."""
    first = _problem(501, [300, 64, 17], H=4, d=128, C=64, dtype="bf16")
    second = _problem(502, [90, 1, 200], H=3, d=64, C=32, dtype="f32")
    for host in (first, second):
        c = host.to("cuda")
        ref_o, ref_h = _with_workspace(c)
        o, h = _no_alloc(c)
        torch.cuda.synchronize()
        tol = tol_for(c.dtype)
        assert rel_err(o, ref_o.double().cpu().numpy()) <= tol
        assert rel_err(h, ref_h.double().cpu().numpy()) <= tol
        oo, oh = oracle_prefill(host)
        lens = [int(x) for x in np.diff(host.cu_host())]
        name = f"no-alloc prefill: lengths {lens} H={c.H} d={c.dk} C={c.chunk} {c.dtype}"
        assert record(name, "o", o, oo) <= tol
        assert record(name, "final_state", h, oh) <= tol


def test_no_alloc_rejects_problems_beyond_the_scratch():
    """Checked on the host before anything is enqueued: no GPU needed."""
    fake = 1 << 20
    total, H, d, C = 1 << 16, 32, 128, 64   # needs far more than the static scratch
    assert kda.kda_chunk_fwd_workspace_size(total, 1, H, d, d, C, "f32") > \
        kda.KDA_NOALLOC_SCRATCH_BYTES
    st = kda.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, None, 1, total, 1, H, d,
                                   d, C, "bf16", fake, None, stream=0, check=False)
    assert st == kda.KDA_ERR_WORKSPACE
