"""GPU parity of the chunkwise prefill (kda_chunk_fwd and the per-step calls)
against the fp64 oracle (token recurrence) and its chunkwise restatement."""
import numpy as np
import pytest
import torch

import gated_delta_rule_124_b200 as kda
from gated_delta_rule_124_b200 import workloads as wl
from oracle import chunkwise
from tests.helpers import oracle_prefill, record, rel_err, tol_for

pytestmark = pytest.mark.gpu


def run_fwd(case, final=True, plan=None):
    """kda_chunk_fwd on the case (its default plan), or kda_chunk_fwd_with_plan."""
    c = case.to("cuda")
    packed = c.cu_seqlens is not None
    B, T = (1, c.total) if packed else (c.B, c.T)
    if plan is None:
        ws = kda.alloc_workspace(c.total, c.N, c.H, c.dk, c.dv, c.chunk, c.dtype)
    else:
        n = kda.kda_chunk_fwd_plan_workspace_size(plan, c.total, c.N, c.H, c.dk, c.dv, c.chunk,
                                                  c.dtype)
        assert n > 0, f"plan {plan} does not apply"
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o = torch.full_like(c.v, float("nan"))
    hN = torch.full((c.N, c.H, c.dk, c.dv), float("nan"), device="cuda") if final else None
    args = (c.q, c.k, c.v, c.g, c.beta, c.initial_state, c.cu_seqlens, B, T, c.N, c.H, c.dk,
            c.dv, c.chunk, c.dtype, o, hN, ws)
    if plan is None:
        kda.kda_chunk_fwd(*args)
    else:
        kda.kda_chunk_fwd_with_plan(plan, *args)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    return o, hN


def check_case(case, heads=None, plan=None, report=False):
    """The case against the fp64 oracle (all heads, or the given ones); with
    `report`, the errors go to the parity report printed after the run."""
    o, hN = run_fwd(case, plan=plan)
    ro, rh = oracle_prefill(case, heads)
    sl = slice(None) if heads is None else list(heads)
    tol = tol_for(case.dtype)
    if report:
        eo = record(case.name, "o", o[:, sl], ro)
        eh = record(case.name, "final_state", hN[:, sl], rh)
    else:
        eo = rel_err(o[:, sl], ro)
        eh = rel_err(hN[:, sl], rh)
    assert eo <= tol and eh <= tol, (case.name, eo, eh)
    return eo, eh


# ---------------------------------------------------------------- configs

# Every configuration at full extent: all sequences, heads and tokens against
# the fp64 oracle (on all host cores), in the launch configuration the
# benchmark times (the default plan of kda_chunk_fwd).

def test_config0_tiny_fp32():
    check_case(wl.prefill_config(0), report=True)


def test_config1_all_heads():
    check_case(wl.prefill_config(1), report=True)


def test_config2_long_all_heads():
    """T = 65536, all 32 heads: each chunk chain is 1024 chunks long, with the
    S operand rounded to bf16 at every chunk."""
    check_case(wl.prefill_config(2), report=True)


def test_config3_varlen_all_heads():
    """16 packed sequences of U[1024, 16384] tokens, all 32 heads."""
    check_case(wl.prefill_config(3), report=True)


# ----------------------------------------------------- shapes and edge cases

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,C", [(32, 32, 16), (64, 32, 32), (32, 128, 64), (128, 64, 16),
                                     (128, 128, 64), (64, 64, 64)])
def test_ragged_lengths(dtype, dk, dv, C):
    """Lengths that are not multiples of the chunk, shorter than one chunk,
    exactly one chunk, and length 1, packed with cu_seqlens."""
    lens = [C * 3 + 5, C - 1, 1, C, 2 * C + 1]
    case = wl.make_prefill(100 + dk + dv + C, lens, H=3, dk=dk, dv=dv, chunk=C, dtype=dtype,
                           varlen=True)
    check_case(case)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_batched_equal_lengths_with_tail(dtype):
    case = wl.make_prefill(5, [200] * 3, H=4, dk=128, dv=128, chunk=64, dtype=dtype)
    check_case(case)


def test_zero_length_sequences_pass_state_through():
    lens = [0, 70, 0, 3, 0]
    case = wl.make_prefill(8, lens, H=2, dk=64, dv=64, chunk=32, dtype="f32", varlen=True)
    o, hN = run_fwd(case)
    ro, rh = oracle_prefill(case)
    assert rel_err(o, ro) <= 1e-4
    assert rel_err(hN, rh) <= 1e-4
    assert torch.equal(hN[0].cpu(), case.initial_state[0])
    assert torch.equal(hN[4].cpu(), case.initial_state[4])


def test_null_initial_state_means_zeros():
    case = wl.make_prefill(9, [150], H=2, dk=128, dv=128, chunk=64, dtype="bf16", init_std=None)
    check_case(case)


def test_strong_decay_is_finite():
    """Gates far below zero (sum of g over a chunk near -300) stay finite."""
    case = wl.make_prefill(10, [256], H=2, dk=128, dv=128, chunk=64, dtype="bf16", g_mu=4.0)
    check_case(case)


def test_split_prefill_composes():
    """Prefill in three calls chained through initial/final state equals one
    call: the state layout is the same on input and output."""
    case = wl.make_prefill(12, [64 * 5 + 17], H=4, dk=128, dv=128, chunk=64, dtype="f32")
    o_full, h_full = run_fwd(case)
    c = case.to("cuda")
    cuts = [0, 64, 64 * 3 + 7, c.total]
    h = c.initial_state
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, h = kda.chunk_fwd(c.q[None, a:b], c.k[None, a:b], c.v[None, a:b], c.g[None, a:b],
                             c.beta[None, a:b], h, chunk=64)
        outs.append(o[0])
    torch.cuda.synchronize()
    assert rel_err(torch.cat(outs), o_full.double().cpu().numpy()) <= 1e-5
    assert rel_err(h, h_full.double().cpu().numpy()) <= 1e-5


def test_final_state_optional_and_in_place():
    case = wl.make_prefill(13, [100, 100], H=2, dk=64, dv=64, chunk=32, dtype="f32")
    c = case.to("cuda")
    ws = kda.alloc_workspace(c.total, 2, 2, 64, 64, 32, "f32")
    o1 = torch.empty_like(c.v)
    kda.kda_chunk_fwd(c.q, c.k, c.v, c.g, c.beta, c.initial_state, None, 2, 100, 2, 2, 64, 64, 32,
                      "f32", o1, None, ws)
    st = c.initial_state.clone()
    o2 = torch.empty_like(c.v)
    kda.kda_chunk_fwd(c.q, c.k, c.v, c.g, c.beta, st, None, 2, 100, 2, 2, 64, 64, 32, "f32", o2,
                      st, ws)
    torch.cuda.synchronize()
    ro, rh = oracle_prefill(case)
    assert rel_err(o1, ro) <= 1e-4 and rel_err(o2, ro) <= 1e-4
    assert rel_err(st, rh) <= 1e-4


def test_bad_cu_seqlens_reported_on_device():
    case = wl.make_prefill(14, [40, 40], H=1, dk=32, dv=32, chunk=16, dtype="f32", varlen=True)
    c = case.to("cuda")
    bad = torch.tensor([0, 50, 40], dtype=torch.int32, device="cuda")  # ends right, not monotone
    ws = kda.alloc_workspace(80, 2, 1, 32, 32, 16, "f32")
    o = torch.empty_like(c.v)
    kda.kda_chunk_fwd(c.q, c.k, c.v, c.g, c.beta, None, bad, 1, 80, 2, 1, 32, 32, 16, "f32", o,
                      None, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_ERR_BAD_SEQLENS
    bad2 = torch.tensor([0, 30, 70], dtype=torch.int32, device="cuda")  # wrong total
    kda.kda_chunk_fwd(c.q, c.k, c.v, c.g, c.beta, None, bad2, 1, 80, 2, 1, 32, 32, 16, "f32", o,
                      None, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_ERR_BAD_SEQLENS
    # a good call on the same workspace clears the word
    kda.kda_chunk_fwd(c.q, c.k, c.v, c.g, c.beta, None, c.cu_seqlens, 1, 80, 2, 1, 32, 32, 16,
                      "f32", o, None, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK


def test_deterministic():
    case = wl.make_prefill(15, [300, 77], H=4, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    o1, h1 = run_fwd(case)
    o2, h2 = run_fwd(case)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


# ------------------------------------------------- one step per call (a1-a4)

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_calls_match_chunkwise_intermediates(dtype):
    lens = [64 * 2 + 9, 30]
    case = wl.make_prefill(16, lens, H=2, dk=128, dv=64, chunk=64, dtype=dtype, varlen=True)
    c = case.to("cuda")
    N, H, dk, dv, C = c.N, c.H, c.dk, c.dv, c.chunk
    tot = c.total
    ws = kda.alloc_workspace(tot, N, H, dk, dv, C, dtype)
    G = torch.empty(tot, H, dk, device="cuda")
    W = torch.empty(tot, H, dk, device="cuda")
    U = torch.empty(tot, H, dv, device="cuda")
    maxc = kda.kda_num_chunks_upper_bound(tot, N, C)
    S = torch.full((maxc, H, dk, dv), float("nan"), device="cuda")
    hN = torch.empty(N, H, dk, dv, device="cuda")
    o = torch.empty_like(c.v)
    args = (c.cu_seqlens, 1, tot, N, H)
    kda.kda_chunk_gate_cumsum(c.g, *args, dk, C, G, ws)
    kda.kda_chunk_intra(c.k, c.v, G, c.beta, *args, dk, dv, C, dtype, W, U, ws)
    Ut = U.clone()
    kda.kda_chunk_inter(c.k, G, W, U, c.initial_state, *args, dk, dv, C, dtype, S, hN, ws)
    kda.kda_chunk_output(c.q, c.k, G, U, S, *args, dk, dv, C, dtype, o, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    f64 = lambda t: t.detach().cpu().double().numpy()
    _, _, inter = chunkwise.forward(f64(case.q), f64(case.k), f64(case.v), f64(case.g),
                                    f64(case.beta), f64(case.initial_state), case.cu_host(),
                                    chunk=C, keep=True)
    cu = case.cu_host()
    gidx = 0
    for s in range(N):
        nch = (lens[s] + C - 1) // C
        for n in range(nch):
            t0 = cu[s] + n * C
            t1 = min(t0 + C, cu[s + 1])
            for h in range(H):
                r = inter[(s, h, n)]
                assert rel_err(G[t0:t1, h], r["G"]) <= 1e-6
                assert rel_err(W[t0:t1, h], r["W"]) <= 1e-4
                assert rel_err(Ut[t0:t1, h], r["Ut"]) <= 1e-4
                assert rel_err(U[t0:t1, h], r["U"]) <= 1e-4
                assert rel_err(S[gidx + n, h], r["S_in"]) <= 1e-5
                assert rel_err(o[t0:t1, h], r["O"]) <= tol_for(dtype)
        gidx += nch
    ro, rh = oracle_prefill(case)
    assert rel_err(o, ro) <= tol_for(dtype)
    assert rel_err(hN, rh) <= 1e-4


def test_mixed_fast_and_exact_chunks():
    """One chunk with extreme decay (its per-channel log-decay range exceeds
    the tensor-core factorisation's headroom, so it is evaluated exactly)
    between ordinary chunks: the state must carry across both kinds."""
    case = wl.make_prefill(17, [64 * 4 + 10], H=2, dk=128, dv=128, chunk=64, dtype="bf16")
    case.g[64:128] *= 6.0
    check_case(case)


@pytest.mark.parametrize("lens", [[1], [63], [65], [1, 1, 1], [0, 64, 0, 129, 7],
                                  [300, 2, 700, 64, 63]])
def test_varlen_edge_lengths_bf16_d128(lens):
    """Packed sequences with lengths around the chunk size, including empty
    and single-token sequences, on the bf16 d = 128 chunk-64 path."""
    case = wl.make_prefill(200 + sum(lens), lens, H=3, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    check_case(case)


# ----------------------------- every prefill plan on the same problems
# bf16, d = 128, chunk 64 runs as the chunk-parallel + per-chain pair of
# tensor-core kernels ("split"), the same pair co-scheduled in one launch
# ("overlap"), or on the CUDA-core kernels ("simt"); kda_chunk_fwd_with_plan
# chooses one explicitly.

PATH_CASES = {
    "varlen": lambda: wl.make_prefill(301, [300, 77, 1, 128], H=4, dk=128, dv=128, chunk=64,
                                      dtype="bf16", varlen=True),
    "empty_seqs": lambda: wl.make_prefill(302, [0, 64, 0, 129, 7], H=3, dk=128, dv=128,
                                          chunk=64, dtype="bf16", varlen=True),
    "batched_tail": lambda: wl.make_prefill(303, [200] * 3, H=4, dk=128, dv=128, chunk=64,
                                            dtype="bf16"),
    "no_initial_state": lambda: wl.make_prefill(304, [150, 70], H=2, dk=128, dv=128, chunk=64,
                                                dtype="bf16", varlen=True, init_std=None),
    "strong_decay": lambda: wl.make_prefill(305, [256], H=2, dk=128, dv=128, chunk=64,
                                            dtype="bf16", g_mu=4.0),
}


@pytest.mark.parametrize("plan", ["split", "overlap", "simt"])
@pytest.mark.parametrize("name", sorted(PATH_CASES))
def test_every_plan_matches_oracle(plan, name):
    check_case(PATH_CASES[name](), plan=plan)


@pytest.mark.parametrize("plan", ["split", "overlap"])
def test_tc_plans_mixed_fast_and_exact_chunks(plan):
    case = wl.make_prefill(306, [64 * 4 + 10], H=2, dk=128, dv=128, chunk=64, dtype="bf16")
    case.g[64:128] *= 6.0
    check_case(case, plan=plan)


def test_plan_that_does_not_apply_is_unsupported():
    """A tensor-core plan for an fp32 problem: KDA_ERR_UNSUPPORTED, and its
    workspace size is 0."""
    case = wl.make_prefill(312, [100], H=2, dk=64, dv=64, chunk=32, dtype="f32").to("cuda")
    assert kda.kda_chunk_fwd_plan_workspace_size("split", case.total, 1, 2, 64, 64, 32,
                                                 "f32") == 0
    ws = kda.alloc_workspace(case.total, 1, 2, 64, 64, 32, "f32")
    o = torch.empty_like(case.v)
    st = kda.kda_chunk_fwd_with_plan("split", case.q, case.k, case.v, case.g, case.beta, None,
                                     None, 1, case.total, 1, 2, 64, 64, 32, "f32", o, None, ws,
                                     check=False)
    assert st == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("lengths", [[640, 333], [64 * 40, 1, 64 * 7 + 5, 0, 200]])
def test_overlap_and_split_identical(lengths):
    """The co-scheduled launch runs the same device code as the two-launch
    split, only interleaved: identical bits."""
    case = wl.make_prefill(310, lengths, H=3, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    o1, h1 = run_fwd(case, plan="split")
    o2, h2 = run_fwd(case, plan="overlap")
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_overlap_repeated_calls_same_workspace():
    """Ready flags are reset by every call: back-to-back calls on one
    workspace give identical results."""
    case = wl.make_prefill(311, [500, 64 * 9], H=4, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    c = case.to("cuda")
    ws = torch.empty(kda.kda_chunk_fwd_plan_workspace_size("overlap", c.total, c.N, c.H, 128,
                                                           128, 64, "bf16"),
                     dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        o = torch.empty_like(c.v)
        hN = torch.empty(c.N, c.H, 128, 128, device="cuda")
        kda.kda_chunk_fwd_with_plan("overlap", c.q, c.k, c.v, c.g, c.beta, c.initial_state,
                                    c.cu_seqlens, 1, c.total, c.N, c.H, 128, 128, 64, "bf16", o,
                                    hN, ws)
        outs.append((o, hN))
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    for o, hN in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(hN, outs[0][1])
    ro, rh = oracle_prefill(case)
    assert rel_err(outs[0][0], ro) <= tol_for("bf16")


def test_default_plans():
    """Long chains over few heads -> overlap; short chains, many chains, or
    packed sequences of unknown length -> split; other shapes -> simt."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    f = kda.kda_chunk_fwd_plan
    assert f(65536, 1, 32, 128, 128, 64, "bf16") == kda.KDA_PLAN_OVERLAP
    assert f(65536, 1, 32, 128, 128, 64, "bf16", packed=True) == kda.KDA_PLAN_OVERLAP
    assert f(65536, 2, 16, 128, 128, 64, "bf16", packed=True) == kda.KDA_PLAN_SPLIT
    assert f(4096, 2, 32, 128, 128, 64, "bf16") == kda.KDA_PLAN_SPLIT
    assert f(4096 * sms, sms, 32, 128, 128, 64, "bf16") == kda.KDA_PLAN_SPLIT
    assert f(4096, 2, 32, 128, 128, 64, "f32") == kda.KDA_PLAN_SIMT


def test_split_step_calls_compose():
    """kda_chunk_split_intra then kda_chunk_split_chain is the split plan of
    kda_chunk_fwd: identical bits, and within tolerance of the oracle."""
    case = wl.make_prefill(308, [333, 64, 0, 700], H=3, dk=128, dv=128, chunk=64,
                           dtype="bf16", varlen=True)
    o1, h1 = run_fwd(case, plan="split")
    c = case.to("cuda")
    n = kda.kda_chunk_split_workspace_size(c.total, c.N, c.H)
    assert n == kda.kda_chunk_fwd_workspace_size(c.total, c.N, c.H, 128, 128, 64, "bf16")
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o = torch.full_like(c.v, float("nan"))
    hN = torch.full((c.N, c.H, 128, 128), float("nan"), device="cuda")
    args = (c.cu_seqlens, 1, c.total, c.N, c.H)
    kda.kda_chunk_split_intra(c.q, c.k, c.g, c.beta, *args, ws)
    kda.kda_chunk_split_chain(c.v, c.initial_state, *args, o, hN, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    assert torch.equal(o, o1) and torch.equal(hN, h1)
    ro, rh = oracle_prefill(case)
    assert rel_err(o, ro) <= tol_for("bf16") and rel_err(hN, rh) <= tol_for("bf16")


def test_split_chain_keeps_the_intra_status():
    """A bad cu_seqlens seen by the intra call stays reported after the chain
    call (the chain call does not reset the status word)."""
    case = wl.make_prefill(309, [128, 64], H=2, dk=128, dv=128, chunk=64, dtype="bf16",
                           varlen=True)
    c = case.to("cuda")
    bad = torch.tensor([0, 150, 140], dtype=torch.int32, device="cuda")  # decreasing
    ws = torch.empty(kda.kda_chunk_split_workspace_size(c.total, c.N, c.H), dtype=torch.uint8,
                     device="cuda")
    o = torch.zeros_like(c.v)
    args = (bad, 1, c.total, c.N, c.H)
    kda.kda_chunk_split_intra(c.q, c.k, c.g, c.beta, *args, ws)
    kda.kda_chunk_split_chain(c.v, None, *args, o, None, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_ERR_BAD_SEQLENS


def test_bounded_wait_reports_timeout_and_next_call_is_clean():
    """The device-side error path, without any fault: the overlap plan with
    one chunk's ready flag withheld and the chains' flag waits bounded by
    10 ms.  The chain that needs that chunk gives up, drains its own copies
    and products and records KDA_ERR_TIMEOUT; the next call on the same
    workspace reports KDA_OK and matches the oracle."""
    case = wl.make_prefill(313, [64 * 6 + 5], H=2, dk=128, dv=128, chunk=64, dtype="bf16")
    c = case.to("cuda")
    n = kda.kda_chunk_fwd_plan_workspace_size("overlap", c.total, 1, 2, 128, 128, 64, "bf16")
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(c.v)
    hN = torch.empty(1, 2, 128, 128, device="cuda")
    kda.kda_test_overlap_flag_timeout(c.q, c.k, c.v, c.g, c.beta, c.initial_state, None, 1,
                                      c.total, 1, 2, o, hN, ws, withheld_chunk=2,
                                      withheld_head=1, flag_wait_ns=10_000_000)
    assert kda.kda_get_device_status(ws) == kda.KDA_ERR_TIMEOUT
    kda.kda_chunk_fwd_with_plan("overlap", c.q, c.k, c.v, c.g, c.beta, c.initial_state, None, 1,
                                c.total, 1, 2, 128, 128, 64, "bf16", o, hN, ws)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    ro, rh = oracle_prefill(case)
    assert rel_err(o, ro) <= tol_for("bf16") and rel_err(hN, rh) <= tol_for("bf16")


def test_timeout_hook_rejects_bad_arguments():
    case = wl.make_prefill(314, [200], H=2, dk=128, dv=128, chunk=64, dtype="bf16").to("cuda")
    n = kda.kda_chunk_fwd_plan_workspace_size("overlap", case.total, 1, 2, 128, 128, 64, "bf16")
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(case.v)
    for chunk, head, wait in ((99, 0, 10_000), (0, 2, 10_000), (0, 0, 0), (0, 0, 3 * 10**9)):
        st = kda.kda_test_overlap_flag_timeout(case.q, case.k, case.v, case.g, case.beta, None,
                                               None, 1, case.total, 1, 2, o, None, ws, chunk,
                                               head, wait, check=False)
        assert st == kda.KDA_ERR_INVALID_ARG, (chunk, head, wait)
