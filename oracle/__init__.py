"""Float64 CPU oracle for the causal TTT / linear-attention layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``; never by the library.
It shares no code, table or helper with the CUDA path.
"""
from .grad_ref import ttt_backward_f64  # noqa: F401
from .feature_ref import feature_map_f64, silu_f64, ttt_feature_layer_f64  # noqa: F401
from .ttt_ref import (  # noqa: F401
    binding_loss_f64,
    ttt_chunked_f64,
    ttt_closed_form_f64,
    ttt_recurrence_f64,
)
