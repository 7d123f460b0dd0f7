"""End-to-end call with host buffers: pinned host -> device copies, the
chunked kernels, and the device -> host copy of the output (and state).

The copies are plain asynchronous cudaMemcpy's on the caller's stream issued
through PyTorch; the layer itself runs only in libttt_la.
"""
from __future__ import annotations

import torch

from ._abi import forward_chunked


class DeviceBuffers:
    """Device-side mirrors of one step's inputs and outputs, reused across
    calls so the end-to-end path allocates nothing per step."""

    def __init__(self, q, k, v, eta, device="cuda"):
        self.q = torch.empty(q.shape, dtype=q.dtype, device=device)
        self.k = torch.empty(k.shape, dtype=k.dtype, device=device)
        self.v = torch.empty(v.shape, dtype=v.dtype, device=device)
        self.eta = None if eta is None else torch.empty(eta.shape, dtype=eta.dtype, device=device)
        self.o = torch.empty(v.shape, dtype=v.dtype, device=device)
        self.ws = None


def forward_chunked_host(q, k, v, eta=None, o_host=None, bufs=None, state_host=None, **kw):
    """q, k, v, eta: (pinned) host tensors.  Copies them in, runs
    ttt_la_forward_chunked, copies o (and the final state when state_host is
    given) back into host tensors.  Returns (o_host, bytes_h2d, bytes_d2h).
    Asynchronous with respect to the host until the caller synchronises."""
    if bufs is None:
        bufs = DeviceBuffers(q, k, v, eta)
    bufs.q.copy_(q, non_blocking=True)
    bufs.k.copy_(k, non_blocking=True)
    bufs.v.copy_(v, non_blocking=True)
    h2d = 3 * q.numel() * q.element_size() if q.shape == v.shape else (
        (q.numel() + k.numel()) * q.element_size() + v.numel() * v.element_size())
    if eta is not None:
        bufs.eta.copy_(eta, non_blocking=True)
        h2d += eta.numel() * eta.element_size()
    o, S, _ = forward_chunked(bufs.q, bufs.k, bufs.v, bufs.eta, out=bufs.o,
                              return_state=state_host is not None, **kw)
    if o_host is None:
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    o_host.copy_(o, non_blocking=True)
    d2h = o.numel() * o.element_size()
    if state_host is not None:
        state_host.copy_(S, non_blocking=True)
        d2h += S.numel() * S.element_size()
    return o_host, h2d, d2h
