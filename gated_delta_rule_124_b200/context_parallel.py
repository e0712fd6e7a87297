"""Context-parallel prefill: one long sequence split over ranks by token ranges.

The state recurrence is affine in the state: over a segment of tokens,
``S_out = M S_in + B`` where ``M`` (dk x dk) is the product of the segment's
transitions ``(I - beta k k^T) Diag(alpha)`` and ``B`` (dk x dv) is the state
the segment builds from a zero state.  Each rank computes its segment's
``(M, B)`` (``kda_chunk_state_maps``: one intra-chunk pass and two chain
passes without outputs -- from zero with the values, and from the identity
with zero values; shapes outside that call: two library prefills), the ranks
exchange them (one all-gather; CPU copies over a gloo group), each rank folds
the maps of the ranks before it into its entry state
(``kda_fold_segment_states``), and a last prefill of its segment from that
state gives its outputs.  Kimi Linear (aiwiki.ai), "The constrained DPLR form
and the chunkwise algorithm": recurrent between chunks -- here between
segments, whose composition is associative.

The backward runs the same way in reverse.  The state gradient's recurrence
does not involve the state, so over a segment ``dS_in = M^T dS_out + c`` with
``c`` the entry-state gradient the segment's own outputs produce (the
library's backward with a zero exit gradient); one exchange of ``(M, B, c)``
gives every rank its entry state (forward fold) and its exit-state gradient
(reverse fold), and a last backward of the segment with both gives its token
gradients.

The local steps are injectable (``prefill``, ``backward``, ``maps``, ``fold``)
so that the exchange logic can be exercised with other implementations of the
same steps (the tests use the fp64 oracle on CPU ranks).
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import kda as _kda

# prefill(q, k, v, g, beta, initial_state) -> (o, final_state); tensors
# [B, T, H, d], states [B, H, dk, dv] fp32.
Prefill = Callable[..., tuple]


def _library_prefill(q, k, v, g, beta, initial_state):
    return _kda.chunk_fwd(q, k, v, g, beta, initial_state=initial_state, chunk=64,
                          output_final_state=True)


# backward(q, k, v, g, beta, initial_state, dout, dfinal_state) ->
# (dq, dk, dv, dg, dbeta, dinitial_state); tensors [B, T, H, d] as above.
Backward = Callable[..., tuple]


def _library_backward(q, k, v, g, beta, initial_state, dout, dfinal_state):
    return _kda.chunk_bwd(q, k, v, g, beta, dout, initial_state, dfinal_state)


def _prefill_maps(q, k, v, g, beta, prefill: Prefill):
    """(M, Bm) of one segment from two prefills: Bm from a zero state; M from
    the identity with zero values (dv = dk for that run)."""
    B, T, H, dk = q.shape
    _, bm = prefill(q, k, v, g, beta, None)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
    zero_v = torch.zeros(B, T, H, dk, dtype=v.dtype, device=v.device)
    _, m = prefill(q, k, zero_v, g, beta, eye)
    return m, bm


def _library_maps(q, k, v, g, beta):
    """(M, Bm) of one segment from the library: kda_chunk_state_maps for bf16,
    dk = dv = 128 (no outputs written), else two library prefills."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if not (q.dtype == torch.bfloat16 and dk == 128 and dv == 128 and q.is_cuda):
        return _prefill_maps(q, k, v, g, beta, _library_prefill)
    f32 = dict(dtype=torch.float32, device=q.device)
    m = torch.empty(B, H, dk, dk, **f32)
    bm = torch.empty(B, H, dk, dv, **f32)
    ws = torch.empty(_kda.kda_chunk_split_workspace_size(B * T, B, H), dtype=torch.uint8,
                     device=q.device)
    flat = lambda x: x.reshape(B * T, *x.shape[2:]).contiguous()  # noqa: E731
    _kda.kda_chunk_state_maps(flat(q), flat(k), flat(v), flat(g), flat(beta), None, B, T, B, H,
                              m, bm, ws)
    return m, bm


def segment_maps(q, k, v, g, beta, prefill: Prefill | None = None):
    """(M [B, H, dk, dk], Bm [B, H, dk, dv]) of one segment: S_out = M S_in + Bm.
    With a `prefill` given, from two calls of it; else from the library."""
    if prefill is not None:
        return _prefill_maps(q, k, v, g, beta, prefill)
    return _library_maps(q, k, v, g, beta)


# fold(M [R, B, H, dk, dk], Bm [R, B, H, dk, dv], S0 [B, H, dk, dv], reverse) ->
# (each [R, B, H, dk, dv], final [B, H, dk, dv]); see kda_fold_segment_states.
Fold = Callable[..., tuple]


def library_fold(M, Bm, S0, reverse=False):
    R, B, H, dk, _ = M.shape
    dv = Bm.shape[-1]
    each = torch.empty(R, B, H, dk, dv, dtype=torch.float32, device=M.device)
    final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=M.device)
    _kda.kda_fold_segment_states(M.contiguous(), Bm.contiguous(), S0.contiguous(), R, B, H, dk,
                                 dv, reverse, each, final)
    return each, final


def entry_states(maps: Sequence[tuple], initial_state, fold: Fold = library_fold):
    """Entry state of every segment and the final state: S_0 = initial_state,
    S_{r+1} = M_r S_r + B_r."""
    M = torch.stack([m for m, _ in maps])
    Bm = torch.stack([b for _, b in maps])
    each, final = fold(M, Bm, initial_state, False)
    return list(each), final


def _all_gather(packed, group):
    """All-gather of this rank's packed maps; over a gloo group the exchange
    goes through CPU copies."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    cpu = dist.get_backend(group) == "gloo" and packed.is_cuda
    src = packed.cpu() if cpu else packed
    gathered = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(gathered, src, group=group)
    return [x.to(packed.device) for x in gathered] if cpu else gathered


def context_parallel_prefill(q, k, v, g, beta, initial_state=None, group=None,
                             prefill: Prefill = _library_prefill, maps=None,
                             fold: Fold = library_fold):
    """This rank's outputs and the final state of the whole sequence.

    q, k, g [B, T_r, H, dk], v [B, T_r, H, dv], beta [B, T_r, H]: this rank's
    token range (ranks in token order); initial_state [B, H, dk, dv] or None
    (zeros), the same on every rank.  One all-gather over `group` (the default
    process group when None).  `maps` (q, k, v, g, beta) -> (M, Bm): the
    segment's maps (default: from the library when `prefill` is the library's,
    else from two calls of `prefill`)."""
    import torch.distributed as dist
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    if initial_state is None:
        initial_state = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if maps is None:
        maps = (_library_maps if prefill is _library_prefill
                else lambda *a: _prefill_maps(*a, prefill))
    m, bm = maps(q, k, v, g, beta)
    rank = dist.get_rank(group)
    packed = torch.cat([m.reshape(B, H, -1), bm.reshape(B, H, -1)], dim=-1).contiguous()
    gathered = _all_gather(packed, group)
    mlist = [(x[..., :dk * dk].reshape(B, H, dk, dk), x[..., dk * dk:].reshape(B, H, dk, dv))
             for x in gathered]
    entries, final = entry_states(mlist, initial_state, fold)
    o, _ = prefill(q, k, v, g, beta, entries[rank].contiguous())
    return o, final


def exit_gradients(maps: Sequence[tuple], offsets: Sequence, dfinal_state,
                   fold: Fold = library_fold):
    """Gradient of every segment's exit state and of the initial state:
    dS_out of the last segment = dfinal_state, dS_out of segment r - 1 =
    dS_in of segment r = M_r^T dS_out_r + c_r."""
    M = torch.stack([m for m, _ in maps])
    C = torch.stack(list(offsets))
    each, g = fold(M, C, dfinal_state, True)
    return list(each), g


def context_parallel_backward(q, k, v, g, beta, dout, initial_state=None, dfinal_state=None,
                              group=None, prefill: Prefill = _library_prefill,
                              backward: Backward = _library_backward, maps=None,
                              fold: Fold = library_fold):
    """Gradients for this rank's tokens of sum(o * dout) + sum(final_state *
    dfinal_state) over the whole sequence, and of the initial state.

    Arguments as in context_parallel_prefill, plus dout [B, T_r, H, dv] for this
    rank's outputs and dfinal_state [B, H, dk, dv] (the same on every rank, or
    None).  Returns (dq, dk, dv, dg, dbeta, dinitial_state); dinitial_state is
    the whole sequence's and the same on every rank.  One all-gather."""
    import torch.distributed as dist
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    f32 = dict(dtype=torch.float32, device=q.device)
    if initial_state is None:
        initial_state = torch.zeros(B, H, dk, dv, **f32)
    if dfinal_state is None:
        dfinal_state = torch.zeros(B, H, dk, dv, **f32)
    if maps is None:
        maps = (_library_maps if prefill is _library_prefill
                else lambda *a: _prefill_maps(*a, prefill))
    m, bm = maps(q, k, v, g, beta)
    c = backward(q, k, v, g, beta, None, dout, None)[5]
    rank = dist.get_rank(group)
    packed = torch.cat([m.reshape(B, H, -1), bm.reshape(B, H, -1),
                        c.reshape(B, H, -1).to(torch.float32)], dim=-1).contiguous()
    gathered = _all_gather(packed, group)
    n1, n2 = dk * dk, dk * dk + dk * dv
    mlist = [(x[..., :n1].reshape(B, H, dk, dk), x[..., n1:n2].reshape(B, H, dk, dv))
             for x in gathered]
    offsets = [x[..., n2:].reshape(B, H, dk, dv) for x in gathered]
    entries, _ = entry_states(mlist, initial_state, fold)
    exits, dh0 = exit_gradients(mlist, offsets, dfinal_state, fold)
    dq, dk_, dv_, dg, db, _ = backward(q, k, v, g, beta, entries[rank].contiguous(), dout,
                                       exits[rank].contiguous())
    return dq, dk_, dv_, dg, db, dh0
