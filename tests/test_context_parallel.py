"""Context-parallel prefill (gated_delta_rule_124_b200.context_parallel): the
exchange and the affine fold, with 2 gloo ranks on the CPU and the fp64 oracle
as each rank's local prefill; on the GPU (marked) the same fold with the
library's kernels over simulated ranks, and the chunked-prefill -> decode
state hand-off."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_124_b200 import context_parallel as cp
from gated_delta_rule_124_b200 import workloads as wl
from tests.helpers import rel_err


def _oracle_prefill(q, k, v, g, beta, initial_state):
    """fp64 oracle as the per-rank prefill (CPU tensors in, float32 out)."""
    o, hN = oracle.forward(q, k, v, g, beta, initial_state)
    return torch.from_numpy(o).float(), torch.from_numpy(hN).float()


def _oracle_backward(q, k, v, g, beta, initial_state, dout, dfinal_state):
    """fp64 gradient oracle as the per-rank backward ([B, T, H, d] tensors)."""
    from oracle import backward as obwd
    B, T, H = q.shape[:3]
    flat = lambda x: None if x is None else x.reshape(B * T, H, *x.shape[3:])  # noqa: E731
    h0 = (torch.zeros(B, H, q.shape[-1], v.shape[-1]) if initial_state is None
          else initial_state)
    r = obwd.backward(flat(q), flat(k), flat(v), flat(g), flat(beta), h0, flat(dout),
                      dfinal_state, np.arange(B + 1) * T)
    shp = (q.shape, k.shape, v.shape, g.shape, beta.shape, h0.shape)
    return tuple(torch.from_numpy(x).float().reshape(s) for x, s in zip(r, shp))


def _host_fold(M, Bm, S0, reverse=False):
    """The fold written out step by step on the host in fp64 (the test's own
    composition of the maps; the product's fold is the library kernel)."""
    M, Bm, S = M.double(), Bm.double(), S0.double()
    R = M.shape[0]
    each = [None] * R
    for step in range(R):
        r = R - 1 - step if reverse else step
        each[r] = S.float()
        S = (M[r].transpose(-1, -2) if reverse else M[r]) @ S + Bm[r]
    return torch.stack(each), S.float()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(T=96, B=2, H=2, d=16, seed=21):
    c = wl.make_prefill(seed, [T] * B, H=H, dk=d, dv=d, chunk=16, dtype="f32")
    sh = lambda x, last: x.reshape(B, T, H, *last)  # noqa: E731
    return (c, sh(c.q, (d,)), sh(c.k, (d,)), sh(c.v, (d,)), sh(c.g, (d,)), sh(c.beta, ()),
            c.initial_state)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c, q, k, v, g, beta, h0 = _case()
        T = q.shape[1]
        a, b = rank * T // world, (rank + 1) * T // world
        o, hN = cp.context_parallel_prefill(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b],
                                            beta[:, a:b], h0, prefill=_oracle_prefill,
                                            fold=_host_fold)
        out[rank] = (o.numpy(), hN.numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_match_the_whole_sequence():
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    c, q, k, v, g, beta, h0 = _case()
    ro, rh = oracle.forward(q, k, v, g, beta, h0)
    o = np.concatenate([out[0][0], out[1][0]], axis=1)
    assert rel_err(o, ro) <= 1e-5
    for r in range(2):
        assert rel_err(out[r][1], rh) <= 1e-5


def _bwd_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c, q, k, v, g, beta, h0 = _case(T=48)
        gen = torch.Generator().manual_seed(3)
        do = torch.randn(q.shape[0], 48, q.shape[2], v.shape[-1], generator=gen)
        dfin = torch.randn(h0.shape, generator=gen)
        T = q.shape[1]
        a, b = rank * T // world, (rank + 1) * T // world
        grads = cp.context_parallel_backward(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b],
                                             beta[:, a:b], do[:, a:b], h0, dfin,
                                             prefill=_oracle_prefill, backward=_oracle_backward,
                                             fold=_host_fold)
        out[rank] = tuple(x.numpy() for x in grads)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_backward_matches_the_whole_sequence():
    """Context-parallel backward over 2 gloo ranks (oracle as each rank's
    prefill and backward) against the oracle's gradients of the whole
    sequence."""
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_bwd_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    c, q, k, v, g, beta, h0 = _case(T=48)
    gen = torch.Generator().manual_seed(3)
    do = torch.randn(q.shape[0], 48, q.shape[2], v.shape[-1], generator=gen)
    dfin = torch.randn(h0.shape, generator=gen)
    ref = _oracle_backward(q, k, v, g, beta, h0, do, dfin)
    for i, name in enumerate(("dq", "dk", "dv", "dg", "dbeta")):
        x = np.concatenate([out[0][i], out[1][i]], axis=1)
        assert rel_err(x, ref[i].numpy()) <= 1e-5, name
    for r in range(2):
        assert rel_err(out[r][5], ref[5].numpy()) <= 1e-5


def test_fold_of_segment_maps_is_the_recurrence():
    """entry_states over oracle-computed maps reproduces the states at the
    segment boundaries (pure host arithmetic)."""
    c, q, k, v, g, beta, h0 = _case(T=60)
    cuts = [0, 13, 40, 60]
    maps = [cp.segment_maps(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b],
                            _oracle_prefill) for a, b in zip(cuts, cuts[1:])]
    entries, final = cp.entry_states(maps, h0, _host_fold)
    for i, a in enumerate(cuts[:-1]):
        if a == 0:
            ref = h0.numpy()
        else:
            _, ref = oracle.forward(q[:, :a], k[:, :a], v[:, :a], g[:, :a], beta[:, :a], h0)
        assert rel_err(entries[i], ref) <= 1e-5
    _, rh = oracle.forward(q, k, v, g, beta, h0)
    assert rel_err(final, rh) <= 1e-5


@pytest.mark.gpu
def test_simulated_ranks_on_the_gpu():
    """Four segments of one 1024-token sequence through the library's kernels:
    maps, fold, finishing prefills."""
    c = wl.make_prefill(22, [1024, 1024], H=4, dk=128, dv=128, chunk=64, dtype="bf16")
    B, T, H, d = 2, 1024, 4, 128
    sh = lambda x, last: x.reshape(B, T, H, *last).cuda()  # noqa: E731
    q, k, v, g = (sh(x, (d,)) for x in (c.q, c.k, c.v, c.g))
    beta, h0 = sh(c.beta, ()), c.initial_state.cuda()
    cuts = [0, 320, 512, 900, 1024]
    segs = list(zip(cuts, cuts[1:]))
    maps = [cp.segment_maps(q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                            v[:, a:b].contiguous(), g[:, a:b].contiguous(),
                            beta[:, a:b].contiguous()) for a, b in segs]
    entries, final = cp.entry_states(maps, h0)
    outs = []
    for (a, b), s_in in zip(segs, entries):
        o, _ = cp._library_prefill(q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                   v[:, a:b].contiguous(), g[:, a:b].contiguous(),
                                   beta[:, a:b].contiguous(), s_in.contiguous())
        outs.append(o)
    o = torch.cat(outs, dim=1)
    ro, rh = oracle.forward(c.q.reshape(B, T, H, d), c.k.reshape(B, T, H, d),
                            c.v.reshape(B, T, H, d), c.g.reshape(B, T, H, d),
                            c.beta.reshape(B, T, H), c.initial_state)
    assert rel_err(o, ro) <= 2e-2 and rel_err(final, rh) <= 2e-2


@pytest.mark.gpu
def test_chunked_prefill_then_decode_hands_the_state_over():
    """Prefill in three pieces (each from the previous piece's final state),
    then decode steps on that state: the same as the oracle's one pass."""
    import gated_delta_rule_124_b200 as kda
    T, H, d = 300, 2, 128
    c = wl.make_prefill(23, [T + 5], H=H, dk=d, dv=d, chunk=64, dtype="bf16")
    cd = c.to("cuda")
    state = cd.initial_state
    outs = []
    for a, b in ((0, 77), (77, 200), (200, T)):
        sl = lambda x: x[a:b].unsqueeze(0).clone()  # noqa: E731  (16-byte aligned copies)
        o, state = kda.chunk_fwd(sl(cd.q), sl(cd.k), sl(cd.v), sl(cd.g), sl(cd.beta),
                                 initial_state=state)
        outs.append(o[0])
    dec = []
    for t in range(T, T + 5):
        one = lambda x: x[t:t + 1].clone()  # noqa: E731
        dec.append(kda.decode_step(one(cd.q), one(cd.k), one(cd.v), one(cd.g), one(cd.beta),
                                   state)[0])
    torch.cuda.synchronize()
    ro, rh = oracle.forward(c.q, c.k, c.v, c.g, c.beta, c.initial_state)
    assert rel_err(torch.cat(outs), ro[:T]) <= 2e-2
    assert rel_err(torch.stack(dec), ro[T:]) <= 2e-2
    assert rel_err(state[0], rh[0]) <= 2e-2


@pytest.mark.gpu
def test_simulated_ranks_backward_on_the_gpu():
    """The context-parallel backward over three segments of two 600-token
    sequences with the library's prefill and backward, against the oracle's
    gradients of the whole sequences."""
    c = wl.make_prefill(24, [600, 600], H=2, dk=64, dv=64, chunk=64, dtype="f32")
    B, T, H, d = 2, 600, 2, 64
    sh = lambda x, last: x.reshape(B, T, H, *last).cuda()  # noqa: E731
    q, k, v, g = (sh(x, (d,)) for x in (c.q, c.k, c.v, c.g))
    beta, h0 = sh(c.beta, ()), c.initial_state.cuda()
    gen = torch.Generator().manual_seed(4)
    do = torch.randn(B, T, H, d, generator=gen)
    dfin = torch.randn(B, H, d, d, generator=gen)
    cuts = [0, 200, 450, 600]
    segs = list(zip(cuts, cuts[1:]))
    part = lambda x, a, b: x[:, a:b].contiguous()  # noqa: E731
    maps, offs = [], []
    for a, b in segs:
        args = [part(x, a, b) for x in (q, k, v, g, beta)]
        maps.append(cp.segment_maps(*args))
        offs.append(cp._library_backward(*args, None, part(do.cuda(), a, b), None)[5])
    entries, _ = cp.entry_states(maps, h0)
    exits, dh0 = cp.exit_gradients(maps, offs, dfin.cuda())
    grads = []
    for (a, b), s_in, d_out in zip(segs, entries, exits):
        args = [part(x, a, b) for x in (q, k, v, g, beta)]
        grads.append(cp._library_backward(*args, s_in.contiguous(), part(do.cuda(), a, b),
                                          d_out.contiguous()))
    ref = _oracle_backward(c.q.reshape(B, T, H, d), c.k.reshape(B, T, H, d),
                           c.v.reshape(B, T, H, d), c.g.reshape(B, T, H, d),
                           c.beta.reshape(B, T, H), c.initial_state, do, dfin)
    for i, name in enumerate(("dq", "dk", "dv", "dg", "dbeta")):
        x = torch.cat([gr[i] for gr in grads], dim=1)
        assert rel_err(x, ref[i].numpy()) <= 1e-3, name
    assert rel_err(dh0, ref[5].numpy()) <= 1e-3


def test_reverse_fold_gives_the_boundary_state_gradients():
    """exit_gradients over oracle maps and oracle state-gradient offsets
    reproduces the gradient of the state at every segment boundary (the
    oracle's initial-state gradient of the suffix after that boundary) and of
    the initial state (pure host arithmetic)."""
    c, q, k, v, g, beta, h0 = _case(T=50)
    gen = torch.Generator().manual_seed(8)
    do = torch.randn(q.shape[0], 50, q.shape[2], v.shape[-1], generator=gen)
    dfin = torch.randn(h0.shape, generator=gen)
    cuts = [0, 11, 30, 50]
    segs = list(zip(cuts, cuts[1:]))
    part = lambda x, a, b: x[:, a:b]  # noqa: E731
    maps = [cp.segment_maps(*(part(x, a, b) for x in (q, k, v, g, beta)), _oracle_prefill)
            for a, b in segs]
    offs = [_oracle_backward(*(part(x, a, b) for x in (q, k, v, g, beta)), None,
                             part(do, a, b), None)[5] for a, b in segs]
    exits, dh0 = cp.exit_gradients(maps, offs, dfin, _host_fold)
    entries, _ = cp.entry_states(maps, h0, _host_fold)
    for i, (a, b) in enumerate(segs):
        if b == 50:
            ref = dfin.numpy()
        else:
            ref = _oracle_backward(*(part(x, b, 50) for x in (q, k, v, g, beta)),
                                   entries[i + 1], part(do, b, 50), dfin)[5].numpy()
        assert rel_err(exits[i], ref) <= 1e-5, i
    assert rel_err(dh0, _oracle_backward(q, k, v, g, beta, h0, do, dfin)[5].numpy()) <= 1e-5


@pytest.mark.gpu
def test_state_maps_from_the_library_match_the_oracle_maps():
    """kda_chunk_state_maps (one intra pass, two chain passes without outputs)
    against the maps the fp64 oracle's two prefills give, on two 200-token
    sequences (three full chunks and a ragged tail)."""
    B, T, H, d = 2, 200, 2, 128
    c = wl.make_prefill(25, [T] * B, H=H, dk=d, dv=d, chunk=64, dtype="bf16")
    sh = lambda x, last: x.reshape(B, T, H, *last)  # noqa: E731
    host = [sh(c.q, (d,)), sh(c.k, (d,)), sh(c.v, (d,)), sh(c.g, (d,)), sh(c.beta, ())]
    m, bm = cp.segment_maps(*(x.cuda() for x in host))
    rm, rb = cp.segment_maps(*host, _oracle_prefill)
    assert rel_err(m.cpu(), rm.numpy()) <= 2e-2
    assert rel_err(bm.cpu(), rb.numpy()) <= 2e-2


@pytest.mark.gpu
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (32, 64)])
@pytest.mark.parametrize("reverse", [False, True])
def test_fold_kernel_matches_the_host_fold(dk, dv, reverse):
    """kda_fold_segment_states against the fold written out in fp64, five
    segments of random maps (contractive M, so the states stay bounded)."""
    gen = torch.Generator().manual_seed(31 + dk + dv + reverse)
    R, N, H = 5, 2, 3
    M = torch.randn(R, N, H, dk, dk, generator=gen) / dk ** 0.5
    Bm = torch.randn(R, N, H, dk, dv, generator=gen)
    S0 = torch.randn(N, H, dk, dv, generator=gen)
    each, fin = cp.library_fold(M.cuda(), Bm.cuda(), S0.cuda(), reverse)
    re, rf = _host_fold(M, Bm, S0, reverse)
    assert rel_err(each.cpu(), re.numpy()) <= 1e-5
    assert rel_err(fin.cpu(), rf.numpy()) <= 1e-5


@pytest.mark.gpu
def test_fold_of_no_segments_returns_the_initial_state():
    S0 = torch.randn(2, 2, 64, 64).cuda()
    M = torch.zeros(0, 2, 2, 64, 64).cuda()
    each, fin = cp.library_fold(M, torch.zeros(0, 2, 2, 64, 64).cuda(), S0, False)
    assert each.shape[0] == 0 and torch.equal(fin, S0)


def _gpu_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, T, H, d = 2, 512, 2, 128
        c = wl.make_prefill(26, [T] * B, H=H, dk=d, dv=d, chunk=64, dtype="bf16")
        a, b = rank * T // world, (rank + 1) * T // world
        part = lambda x, last: x.reshape(B, T, H, *last)[:, a:b].contiguous().cuda()  # noqa: E731
        o, hN = cp.context_parallel_prefill(part(c.q, (d,)), part(c.k, (d,)), part(c.v, (d,)),
                                            part(c.g, (d,)), part(c.beta, ()),
                                            c.initial_state.cuda())
        torch.cuda.synchronize()
        out[rank] = (o.float().cpu().numpy(), hN.cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_two_ranks_gloo_with_the_library_on_the_gpu():
    """context_parallel_prefill with its defaults (the library's maps, fold
    and prefill on cuda:0) in two processes exchanging over gloo, against the
    oracle over the whole 512-token sequences.  The ranks' kernels never wait
    on each other: the exchange is a host all-gather between them."""
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.spawn(_gpu_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    B, T, H, d = 2, 512, 2, 128
    c = wl.make_prefill(26, [T] * B, H=H, dk=d, dv=d, chunk=64, dtype="bf16")
    sh = lambda x, last: x.reshape(B, T, H, *last)  # noqa: E731
    ro, rh = oracle.forward(sh(c.q, (d,)), sh(c.k, (d,)), sh(c.v, (d,)), sh(c.g, (d,)),
                            sh(c.beta, ()), c.initial_state)
    o = np.concatenate([out[0][0], out[1][0]], axis=1)
    assert rel_err(o, ro) <= 2e-2
    for r in range(2):
        assert rel_err(out[r][1], rh) <= 2e-2
