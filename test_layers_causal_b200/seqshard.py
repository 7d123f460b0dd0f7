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

The backward has one exchange too.  A run's backward is affine in the
gradients entering its end, and the linear part is the adjoint of the run's
forward map: per head a multiple of the identity,
    (G, H) -> (G, P H - G_run G)      (P = beta^L; without momentum only G),
so each rank
  1. rebuilds its start state as in the forward (maps, all-gather, compose),
  2. runs its backward with no gradient entering its end; the dL/dW_0,
     dL/dM_0 it returns are the run's constant term (B_W, B_M),
  3. all-gathers them (d_v x d_k fp32 per head, one or two),
  4. folds the later runs' adjoint maps onto (dL/dW_T, dL/dM_T) with
     ttt_la_compose_maps (whose elementwise form w - G m + dW, B m + dM
     expresses both steps with per-head scalars),
  5. runs its backward again from that end gradient for dq, dk, dv, deta.
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


def chunked_backward_supported(q, v, beta):
    """Whether ttt_la_backward_chunked takes these shapes: bf16 with d_k == d_v
    in {64, 128} (with or without momentum), fp32 without momentum with d_k,
    d_v multiples of 4 up to 128."""
    dk, dv = q.shape[-1], v.shape[-1]
    if q.dtype == torch.bfloat16:
        return dk == dv and dk in (64, 128)
    return not beta and dk % 4 == 0 and dv % 4 == 0 and dk <= 128 and dv <= 128


def _library_backward(q, k, v, dO, eta, **kw):
    """A run's backward: the chunk-parallel form where the library has it,
    else the recurrent one."""
    if chunked_backward_supported(q, v, kw.get("beta", 0.0)):
        return _abi.backward_chunked(q, k, v, dO, eta, **kw)
    return _abi.backward_recurrent(q, k, v, dO, eta, **kw)


LIBRARY = Backend(
    segment_map=_abi.segment_map,
    compose_maps=_abi.compose_maps,
    forward=lambda q, k, v, eta, **kw: _abi.forward_chunked(q, k, v, eta, **kw),
    backward=_library_backward,
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


def _stack_gb(G, P):
    """[1, B, H, 2] map scalars (G, P) for ttt_la_compose_maps."""
    return torch.stack([G, P], dim=-1).unsqueeze(0).contiguous()


def backward_sequence_sharded(q, k, v, dO, eta=None, *, rank=0, world=1, eta_const=None, beta=0.0, ascent=False,
                              chunk=64, state_in=None, mom_in=None, grad_state=None, grad_mom=None,
                              backend: Backend = LIBRARY):
    """Backward of the layer for this rank's run of every sequence (see
    token_slice).  q, k, v, dO, eta: this run's tokens; state_in, mom_in =
    W_0, M_0 and grad_state, grad_mom = dL/dW_T, dL/dM_T [B,H,d_v,d_k] (the
    same on every rank) or None.  Returns (dq, dk, dv, deta) for this run and
    (dL/dW_0, dL/dM_0) of the whole sequence (identical on every rank; dL/dM_0
    is None without momentum).

    The gradients entering run r's end: G_end_r = dL/dW_T + sum_{r' > r} B_W,r'
    (W's gradient passes a run unchanged plus the run's own do q^T sums), and
    with momentum H_end_r from the adjoint of each later run's map,
        H <- P_r' H - G_r' G_end_r' + B_M,r'      (r' = last run down to r + 1),
    where (G_r', P_r') are the run's map scalars (G and beta^L of
    ttt_la_segment_map) and (B_W,r', B_M,r') the dL/dW_0, dL/dM_0 of run r''s
    backward with no gradient entering its end."""
    kw = dict(eta_const=eta_const, beta=beta, ascent=ascent)
    dW, dM, GB = backend.segment_map(q, k, v, eta, chunk=chunk, **kw)
    dW_all = _all_gather(dW, world)
    dM_all = _all_gather(dM, world) if dM is not None else None
    GB_all = _all_gather(GB, world) if GB is not None else None
    W0, M0 = backend.compose_maps(dW_all[:rank], None if dM_all is None else dM_all[:rank],
                                  None if GB_all is None else GB_all[:rank], state_in, mom_in)
    bk = dict(kw, state_in=W0, mom_in=M0 if beta else None)
    z = backend.backward(q, k, v, dO, eta, **bk)  # this run with no gradient entering its end
    BW_all = _all_gather(z["dW0"], world)
    BM_all = _all_gather(z["dM0"], world) if beta else None

    def g_end(r):  # dL/dW at the end of run r
        return backend.compose_maps(BW_all[r + 1:], None, None, grad_state, None)[0]

    def h_fold(r_stop):  # dL/dM at the end of run r_stop (r_stop = -1: at the start of run 0)
        H = grad_mom if grad_mom is not None else torch.zeros_like(BW_all[0])
        for r2 in range(world - 1, r_stop, -1):
            G2, P2 = GB_all[r2][..., 0], GB_all[r2][..., 1]
            zero = torch.zeros_like(BW_all[0])
            # C = B_M - G G_end, then H = P H + C (the W channel of the map is idle)
            C, _ = backend.compose_maps(zero.unsqueeze(0), zero.unsqueeze(0), _stack_gb(G2, torch.ones_like(P2)),
                                        BM_all[r2], g_end(r2))
            _, H = backend.compose_maps(zero.unsqueeze(0), C.unsqueeze(0), _stack_gb(torch.zeros_like(G2), P2),
                                        zero, H)
        return H

    G_end = g_end(rank)
    H_end = h_fold(rank) if beta else None
    g = backend.backward(q, k, v, dO, eta, grad_state=G_end, grad_mom=H_end, **bk)
    dW0 = backend.compose_maps(BW_all, None, None, grad_state, None)[0]
    dM0 = h_fold(-1) if beta else None
    return g["dq"], g["dk"], g["dv"], g["deta"], dW0, dM0
