"""End-to-end call with host buffers: the library's pipelined host entry
point (ttt_la_forward_chunked_host) copies the inputs in piece by piece, runs
the chunked kernel on each piece and copies the outputs back, overlapping the
three on separate streams.  This module only keeps the device staging buffer
between calls and counts the bytes that cross the bus.
"""
from __future__ import annotations

from . import _abi


class HostStaging:
    """Device staging reused across calls (allocated on first use)."""

    def __init__(self):
        self.buf = None


def forward_chunked_host(q, k, v, eta=None, o_host=None, bufs=None, state_host=None, **kw):
    """q, k, v, eta: (pinned) host tensors.  Returns (o_host, bytes_h2d,
    bytes_d2h); the copies and the kernels are queued on the current stream's
    order (complete when it is).  `state_host` receives the final state."""
    if bufs is None:
        bufs = HostStaging()
    kw.pop("workspace", None)
    o, bufs.buf = _abi.forward_chunked_host(q, k, v, eta, out=o_host, state_out=state_host, staging=bufs.buf, **kw)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v, eta, kw.get("state_in"), kw.get("mom_in"))
              if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in (o, state_host) if t is not None)
    return o, h2d, d2h
