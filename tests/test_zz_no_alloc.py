"""The chunked forward for callers that cannot allocate device memory.

Some callers only receive input and output buffers (a plugin inside another
engine, code whose device memory belongs to someone else's pool) and cannot
call cudaMalloc; ttt_la_forward_chunked_noalloc serves them with a fixed
scratch array inside the library.  This test calls it through the C ABI and
checks its output and final state against the allocating entry point on two
calls in a row (the array is reused and keeps the previous call's contents).
It lives in a file of its own that pytest collects last.
"""
import ctypes
import math

import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(B, H, T, d, seed):
    from synth import make_qkv
    q, k, v, z = make_qkv((B, H), T, d, d, seed)
    eta = (torch.sigmoid(z) / math.sqrt(d)).float()
    return [x.cuda().contiguous() for x in (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), eta)]


def _call_noalloc(q, k, v, eta, chunk, segments, o, S):
    from test_layers_causal_b200 import _abi
    a = _abi._seq_args(q, k, v, eta, None, 0.0, False, chunk, segments, None, None, o, S, None)
    a.workspace, a.workspace_bytes = None, 0  # ignored by this entry point
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _abi.lib().ttt_la_forward_chunked_noalloc(ctypes.byref(a), st)


def _rel(x, ref):
    x, ref = x.float(), ref.float()
    return float((x - ref).norm() / ref.norm())


@pytest.mark.parametrize("d,chunk,T,segments", [(64, 64, 2000, 4), (128, 128, 1500, 3)])
def test_noalloc_matches_allocating_entry_point(d, chunk, T, segments):
    import test_layers_causal_b200 as ttt
    from test_layers_causal_b200 import _abi
    B, H = 2, 3
    for call, seed in enumerate((11, 12)):  # two calls in a row on the shared array
        q, k, v, eta = _inputs(B, H, T, d, seed)
        assert _abi.workspace_bytes(q, v, chunk=chunk, segments=segments) > 0  # this shape needs scratch
        o_ref, S_ref, _ = ttt.forward_chunked(q, k, v, eta, chunk=chunk, segments=segments)
        o = torch.empty_like(v)
        S = torch.empty(B, H, d, d, device="cuda", dtype=torch.float32)
        code = _call_noalloc(q, k, v, eta, chunk, segments, o, S)
        assert code == 0, _abi.status_string(code)
        torch.cuda.synchronize()
        assert ttt.device_status() == 0
        assert _rel(o, o_ref) <= 2e-2, f"call {call}: o"
        assert _rel(S, S_ref) <= 2e-2, f"call {call}: state"


def test_noalloc_rejects_scratch_beyond_its_array():
    from test_layers_causal_b200 import _abi
    B, H, T, d = 1, 1, 128 * 700, 128
    q, k, v = (torch.zeros(B, H, T, d, device="cuda", dtype=torch.bfloat16) for _ in range(3))
    eta = None
    need = _abi.workspace_bytes(q, v, chunk=128, segments=600)
    assert need > _abi.STATIC_SCRATCH_BYTES
    o = torch.empty_like(v)
    assert _call_noalloc(q, k, v, eta, 128, 600, o, None) == _abi.ERR_SCRATCH_LIMIT
