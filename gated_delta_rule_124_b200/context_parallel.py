"""Context-parallel prefill: one long sequence split over ranks by token ranges.

The state recurrence is affine in the state: over a segment of tokens,
``S_out = M S_in + B`` where ``M`` (dk x dk) is the product of the segment's
transitions ``(I - beta k k^T) Diag(alpha)`` and ``B`` (dk x dv) is the state
the segment builds from a zero state.  Each rank computes its segment's
``(M, B)`` with the library's prefill (``B``: the segment from a zero state;
``M``: the segment with zero values from the identity state, so the carried
state is exactly the product of the transitions), the ranks exchange them
(one all-gather), each rank folds the maps of the ranks before it into its
entry state, and a last prefill of its segment from that state gives its
outputs.  Kimi Linear (aiwiki.ai), "The constrained DPLR form and the
chunkwise algorithm": recurrent between chunks -- here between segments, whose
composition is associative.

Cost: three prefills of the local segment per rank (two independent, one
after the exchange) plus ``R`` small dk x dk products; the exchange carries
``2 x H x dk x max(dk, dv)`` floats per sequence and rank.

The backward runs the same way in reverse.  The state gradient's recurrence
does not involve the state, so over a segment ``dS_in = M^T dS_out + c`` with
``c`` the entry-state gradient the segment's own outputs produce (the
library's backward with a zero exit gradient); one exchange of ``(M, B, c)``
gives every rank its entry state (forward fold) and its exit-state gradient
(reverse fold), and a last backward of the segment with both gives its token
gradients.
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


def segment_maps(q, k, v, g, beta, prefill: Prefill = _library_prefill):
    """(M [B, H, dk, dk], Bm [B, H, dk, dv]) of one segment: S_out = M S_in + Bm."""
    B, T, H, dk = q.shape
    _, bm = prefill(q, k, v, g, beta, None)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
    zero_v = torch.zeros(B, T, H, dk, dtype=v.dtype, device=v.device)
    _, m = prefill(q, k, zero_v, g, beta, eye)
    return m, bm


def entry_states(maps: Sequence[tuple], initial_state):
    """Entry state of every segment and the final state: S_0 = initial_state,
    S_{r+1} = M_r S_r + B_r."""
    s = initial_state
    out = [s]
    for m, bm in maps:
        s = torch.matmul(m, s) + bm
        out.append(s)
    return out[:-1], out[-1]


def context_parallel_prefill(q, k, v, g, beta, initial_state=None, group=None,
                             prefill: Prefill = _library_prefill):
    """This rank's outputs and the final state of the whole sequence.

    q, k, g [B, T_r, H, dk], v [B, T_r, H, dv], beta [B, T_r, H]: this rank's
    token range (ranks in token order); initial_state [B, H, dk, dv] or None
    (zeros), the same on every rank.  One all-gather over `group` (the default
    process group when None)."""
    import torch.distributed as dist
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    if initial_state is None:
        initial_state = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=q.device)
    m, bm = segment_maps(q, k, v, g, beta, prefill)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    packed = torch.cat([m.reshape(B, H, -1), bm.reshape(B, H, -1)], dim=-1).contiguous()
    gathered = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(gathered, packed, group=group)
    maps = [(x[..., :dk * dk].reshape(B, H, dk, dk), x[..., dk * dk:].reshape(B, H, dk, dv))
            for x in gathered]
    entries, final = entry_states(maps, initial_state)
    o, _ = prefill(q, k, v, g, beta, entries[rank].contiguous())
    return o, final


def exit_gradients(maps: Sequence[tuple], offsets: Sequence, dfinal_state):
    """Gradient of every segment's exit state and of the initial state:
    dS_out of the last segment = dfinal_state, dS_out of segment r - 1 =
    dS_in of segment r = M_r^T dS_out_r + c_r."""
    g = dfinal_state
    out = [None] * len(maps)
    for r in range(len(maps) - 1, -1, -1):
        out[r] = g
        g = torch.matmul(maps[r][0].transpose(-1, -2), g) + offsets[r]
    return out, g


def context_parallel_backward(q, k, v, g, beta, dout, initial_state=None, dfinal_state=None,
                              group=None, prefill: Prefill = _library_prefill,
                              backward: Backward = _library_backward):
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
    m, bm = segment_maps(q, k, v, g, beta, prefill)
    c = backward(q, k, v, g, beta, None, dout, None)[5]
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    packed = torch.cat([m.reshape(B, H, -1), bm.reshape(B, H, -1),
                        c.reshape(B, H, -1).to(torch.float32)], dim=-1).contiguous()
    gathered = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(gathered, packed, group=group)
    n1, n2 = dk * dk, dk * dk + dk * dv
    maps = [(x[..., :n1].reshape(B, H, dk, dk), x[..., n1:n2].reshape(B, H, dk, dv))
            for x in gathered]
    offsets = [x[..., n2:].reshape(B, H, dk, dv) for x in gathered]
    entries, _ = entry_states(maps, initial_state)
    exits, dh0 = exit_gradients(maps, offsets, dfinal_state)
    dq, dk_, dv_, dg, db, _ = backward(q, k, v, g, beta, entries[rank].contiguous(), dout,
                                       exits[rank].contiguous())
    return dq, dk_, dv_, dg, db, dh0
