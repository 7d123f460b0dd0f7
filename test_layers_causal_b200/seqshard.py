"""One sequence split over several devices along T, with one exchange step.

Every (b, h) sequence's tokens are cut into contiguous runs, run r on rank r.
A run acts on the carried state as an affine map
    (W, M) -> (W - G M + dW, B M + dM)
(Variant 3 of Table 2 in the thelatestinai.com listing of "Test-Time Training
with KV Binding Is Secretly Linear Attention" carries (W, M); without momentum
G = 0, B = 1 and only dW matters).  So each rank
  1. computes its run's map (ttt_la_segment_map),
  2. all-gathers every rank's map (d_v x d_k fp32 per head, the only
     collective on the data path),
  3. composes the maps of the runs before its own onto (W_0, M_0) into its
     start state, and the maps of all runs into the final state
     (ttt_la_compose_maps),
  4. runs the chunked forward over its run from that start state.
The arithmetic runs in the library; this module only moves tensors and
orders the calls.  The `backend` argument exists so that the orchestration
can be exercised on CPU ranks with a substitute for the library.

The backward (without momentum) has one exchange too.  The gradient with
respect to the state at the end of run r is
    G_end_r = dL/dW_T + sum over later runs r' of B_r',   B_r' = sum_{t in r'} do_t q_t^T,
and B_r is what the backward of run r returns as dL/dW_0 when no gradient
enters its final state.  So each rank
  1. rebuilds its start state as in the forward (maps, all-gather, compose),
  2. runs its backward from a zero final-state gradient to get B_r,
  3. all-gathers the B's (d_v x d_k fp32 per head) and sums the later ones
     onto dL/dW_T (ttt_la_compose_maps with plain maps),
  4. runs its backward again from that end gradient for dq, dk, dv, deta.
dL/dW_0 of the whole sequence is dL/dW_T plus all the B's.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import _abi


def token_slice(T: int, rank: int, world: int) -> slice:
    """Contiguous run of the T tokens owned by `rank` (lengths differ by at
    most one; earlier ranks hold the earlier tokens)."""
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


@dataclasses.dataclass(frozen=True)
class Backend:
    """The operations the split needs (the library by default)."""
    segment_map: object
    compose_maps: object
    forward: object
    backward: object = None


LIBRARY = Backend(
    segment_map=_abi.segment_map,
    compose_maps=_abi.compose_maps,
    forward=lambda q, k, v, eta, **kw: _abi.forward_chunked(q, k, v, eta, **kw),
    backward=lambda q, k, v, dO, eta, **kw: _abi.backward_recurrent(q, k, v, dO, eta, **kw),
)


def _all_gather(t, world):
    if world == 1:
        return t.unsqueeze(0)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous())
    return torch.stack(parts)


def forward_sequence_sharded(q, k, v, eta=None, *, rank=0, world=1, eta_const=None, beta=0.0, ascent=False,
                             chunk=64, state_in=None, mom_in=None, backend: Backend = LIBRARY):
    """q, k, v [B,H,T_r,d], eta [B,H,T_r]: this rank's run of every sequence
    (see token_slice).  state_in / mom_in: W_0, M_0 [B,H,d_v,d_k] (the same on
    every rank) or None.  Returns (o, W_T, M_T): this run's output and the
    state after the whole sequence (identical on every rank; M_T None
    without momentum)."""
    kw = dict(eta_const=eta_const, beta=beta, ascent=ascent, chunk=chunk)
    dW, dM, GB = backend.segment_map(q, k, v, eta, **kw)
    dW_all = _all_gather(dW, world)
    dM_all = _all_gather(dM, world) if dM is not None else None
    GB_all = _all_gather(GB, world) if GB is not None else None
    W0, M0 = backend.compose_maps(dW_all[:rank], None if dM_all is None else dM_all[:rank],
                                  None if GB_all is None else GB_all[:rank], state_in, mom_in)
    o, _, _ = backend.forward(q, k, v, eta, state_in=W0, mom_in=M0 if beta else None, return_state=False, **kw)
    W_T, M_T = backend.compose_maps(dW_all, dM_all, GB_all, state_in, mom_in)
    return o, W_T, (M_T if beta else None)


def backward_sequence_sharded(q, k, v, dO, eta=None, *, rank=0, world=1, eta_const=None, ascent=False, chunk=64,
                              state_in=None, grad_state=None, backend: Backend = LIBRARY):
    """Backward of the layer without momentum for this rank's run of every
    sequence (see token_slice).  q, k, v, dO, eta: this run's tokens;
    state_in = W_0 and grad_state = dL/dW_T [B,H,d_v,d_k] (the same on every
    rank) or None.  Returns (dq, dk, dv, deta) for this run and dL/dW_0 of the
    whole sequence (identical on every rank)."""
    dW, _, _ = backend.segment_map(q, k, v, eta, eta_const=eta_const, beta=0.0, ascent=ascent, chunk=chunk)
    dW_all = _all_gather(dW, world)
    W0, _ = backend.compose_maps(dW_all[:rank], None, None, state_in, None)
    kw = dict(eta_const=eta_const, ascent=ascent, state_in=W0)
    own = backend.backward(q, k, v, dO, eta, **kw)["dW0"]  # B_r = sum over this run of do q^T
    own_all = _all_gather(own, world)
    G_end, _ = backend.compose_maps(own_all[rank + 1:], None, None, grad_state, None)
    g = backend.backward(q, k, v, dO, eta, grad_state=G_end, **kw)
    dW0, _ = backend.compose_maps(own_all, None, None, grad_state, None)
    return g["dq"], g["dk"], g["dv"], g["deta"], dW0
