"""Causal TTT / linear-attention layer for B200 (sm_100a).

The C ABI lives in ``include/ttt_la.h`` and ``libttt_la.so`` (built in-tree by
``python -m test_layers_causal_b200.build``); this package is its thin Python
binding.  Entry points: ``forward_chunked``, ``forward_recurrent``,
``decode_step`` (see ``_abi``) and ``forward_chunked_host`` (host buffers in,
host buffers out, for end-to-end timing).
"""
from ._abi import (  # noqa: F401
    TttError, decode_step, device_status, forward_chunked, forward_recurrent, lib,
    selftest_wait_timeout, set_wait_limit_ns, status_string, version, workspace_bytes,
)
from .host import forward_chunked_host  # noqa: F401
