"""The chunked forward for callers that cannot allocate device memory.

Some callers only receive input and output buffers (a plugin inside another
engine, code whose device memory belongs to someone else's pool) and cannot
call cudaMalloc; ttt_la_forward_chunked_noalloc serves them with a fixed
scratch array inside the library.  This test calls it through the C ABI and
checks its output and final states against the allocating entry point on two
calls in a row, after a larger call has left its own values in the shared
array (the array keeps the previous call's contents).

Where the start states come from a cooperative prefix, both entry points sum
in a fixed order and must agree bit for bit.  With the decoupled look-back a
block starts from whichever predecessor states are already published, so the
fp32 summation order (and, rarely, a bf16 rounding of the output) can differ
between any two runs: there the bound is 1e-3 on the output and 1e-5 on the
fp32 states, far below what stale scratch would produce.
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


def _call_noalloc(q, k, v, eta, chunk, segments, o, S, beta=0.0, M=None):
    from test_layers_causal_b200 import _abi
    a = _abi._seq_args(q, k, v, eta, None, beta, False, chunk, segments, None, None, o, S, M)
    a.workspace, a.workspace_bytes = None, 0  # ignored by this entry point
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _abi.lib().ttt_la_forward_chunked_noalloc(ctypes.byref(a), st)


def _rel(x, ref):
    x, ref = x.float(), ref.float()
    return float((x - ref).norm() / ref.norm())


def _noalloc_outputs(q, k, v, eta, chunk, segments, beta):
    from test_layers_causal_b200 import _abi
    B, H, _, d = q.shape
    o = torch.empty_like(v)
    S = torch.empty(B, H, d, d, device="cuda", dtype=torch.float32)
    M = torch.empty_like(S) if beta else None
    code = _call_noalloc(q, k, v, eta, chunk, segments, o, S, beta, M)
    assert code == 0, _abi.status_string(code)
    return o, S, M


# (d, chunk, B, H, T, segments, beta): look-back without momentum at both
# widths, the cooperative prefix without and with momentum
CASES = [(64, 64, 2, 3, 2000, 4, 0.0), (128, 128, 2, 3, 1500, 3, 0.0), (128, 128, 1, 2, 128 * 40, 20, 0.0),
         (128, 128, 1, 2, 8192, 8, 0.9)]


@pytest.mark.parametrize("d,chunk,B,H,T,segments,beta", CASES)
def test_noalloc_matches_allocating_entry_point(d, chunk, B, H, T, segments, beta):
    import test_layers_causal_b200 as ttt
    from test_layers_causal_b200 import _abi
    plan = ttt.chunked_plan(B, H, T, d, d, chunk=chunk, beta=beta, segments=segments, eta=True)
    assert 0 < plan["workspace_bytes"] <= _abi.STATIC_SCRATCH_BYTES  # this shape needs scratch, and fits
    exact = plan["cooperative"] == 1
    # a larger call first leaves its own totals and flags in the shared array
    big = _inputs(1, 4, 128 * 24, 128, 7)
    _noalloc_outputs(*big, 128, 6, 0.0)
    for call, seed in enumerate((11, 12)):  # two calls in a row on the shared array
        q, k, v, eta = _inputs(B, H, T, d, seed)
        o_ref, S_ref, M_ref = ttt.forward_chunked(q, k, v, eta, beta=beta, chunk=chunk, segments=segments)
        o, S, M = _noalloc_outputs(q, k, v, eta, chunk, segments, beta)
        torch.cuda.synchronize()
        assert ttt.device_status() == 0
        pairs = [(o, o_ref, 1e-3, "o"), (S, S_ref, 1e-5, "state")] + ([(M, M_ref, 1e-5, "mom")] if beta else [])
        for x, ref, tol, name in pairs:
            if exact:
                assert torch.equal(x, ref), f"call {call}: {name} differs from the allocating entry point"
            else:
                assert _rel(x, ref) <= tol, f"call {call}: {name} rel error {_rel(x, ref):.2e}"


def test_noalloc_rejects_scratch_beyond_its_array():
    from test_layers_causal_b200 import _abi
    B, H, T, d = 1, 1, 128 * 700, 128
    q, k, v = (torch.zeros(B, H, T, d, device="cuda", dtype=torch.bfloat16) for _ in range(3))
    eta = None
    need = _abi.workspace_bytes(q, v, chunk=128, segments=600)
    assert need > _abi.STATIC_SCRATCH_BYTES
    o = torch.empty_like(v)
    assert _call_noalloc(q, k, v, eta, 128, 600, o, None) == _abi.ERR_SCRATCH_LIMIT
