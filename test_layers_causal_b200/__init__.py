"""Causal TTT / linear-attention layer for B200 (sm_100a).

The C ABI lives in ``include/ttt_la.h`` and ``libttt_la.so`` (built in-tree by
``python -m test_layers_causal_b200.build``); this package is its thin Python
binding.  Entry points: ``forward_chunked``, ``forward_recurrent``,
``decode_step``, ``segment_map``, ``compose_maps``, ``feature_map`` (the
frozen gated-MLP feature map of keys and queries) and ``forward_chunked_phi``
(feature map, then the chunked forward), ``backward_recurrent`` (the
layer's gradient) (see ``_abi``),
``forward_chunked_host`` (host buffers in, host buffers out, for end-to-end
timing) and ``forward_sequence_sharded`` (one sequence split over ranks along
T, see ``seqshard``).
"""
from ._abi import (  # noqa: F401
    TttError, backward_chunked, backward_recurrent, chunked_plan, compose_maps, decode_step, device_status, feature_map, forward_chunked,
    forward_chunked_phi,
    forward_recurrent, lib, segment_map,
    selftest_wait_timeout, set_wait_limit_ns, status_string, version, workspace_bytes,
)
from .host import forward_chunked_host  # noqa: F401
from .seqshard import backward_sequence_sharded, forward_sequence_sharded, token_slice  # noqa: F401
