"""The debug build (libttt_la_debug.so, compiled with -DTTT_LA_DEBUG) on tiny,
ragged shapes through the C ABI: every hand-indexed access of the chunked
kernels to the workspace, flags and states is checked against the sizes of
the call, and a failed check would record TTT_LA_ERR_DEVICE_CHECK and its
source line instead of touching memory.  Each case covers one scratch
layout -- one segment (none), the decoupled look-back, the wave schedule,
and momentum with its look-back and its cooperative prefix -- and must leave
a clean status word, a clean check line and outputs within the bf16
tolerance of the float64 oracle."""
import ctypes
import math

import pytest
import torch

from synth import make_qkv
from tests.gpu_util import assert_bf16, f64, oracle_forward

pytestmark = pytest.mark.gpu


def _inputs(B, H, T, d, seed):
    q, k, v, z = make_qkv((B, H), T, d, d, seed)
    eta = (torch.sigmoid(z) / math.sqrt(d)).float()
    return [x.cuda().contiguous() for x in (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), eta)]


# (d, chunk, B, H, T, segments, beta, wave tokens): ragged T everywhere
CASES = [
    (64, 64, 1, 2, 100, 1, 0.0, 0),           # one segment: no scratch
    (64, 64, 2, 3, 64 * 9 + 5, 3, 0.0, 0),    # look-back, merged 64 x 64 tiles
    (128, 128, 1, 2, 128 * 7 + 9, 4, 0.0, 0), # look-back, 128-wide tiles
    (128, 128, 1, 2, 128 * 36 - 1, 6, 0.0, 128),  # wave schedule, six waves
    (128, 64, 1, 2, 64 * 30 + 3, 6, 0.0, 64),     # wave schedule, 64-token tiles
    (64, 128, 1, 3, 128 * 45 - 7, 14, 0.0, 128),  # wave schedule, d = 64
    (128, 64, 1, 2, 64 * 9 + 1, 3, 0.9, 0),   # momentum, cooperative prefix
    (64, 64, 16, 16, 64 * 3 + 2, 2, 0.9, 0),  # momentum, look-back (grid beyond one wave)
]


@pytest.mark.parametrize("d,chunk,B,H,T,segments,beta,wave_tokens", CASES)
def test_debug_build_checks_stay_clean(d, chunk, B, H, T, segments, beta, wave_tokens, monkeypatch):
    from test_layers_causal_b200 import _abi
    if wave_tokens:
        monkeypatch.setenv("TTT_LA_WAVE_TOKENS", str(wave_tokens))
    L = _abi.debug_lib()
    assert b"debug checks" in L.ttt_la_version()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L.ttt_la_debug_check_line(st)  # clear whatever an earlier call left
    L.ttt_la_get_last_device_status(st)
    q, k, v, eta = _inputs(B, H, T, d, 300 + d + T)
    S0 = 0.1 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(5)).cuda()
    M0 = 0.1 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(6)).cuda() if beta else None
    o = torch.empty_like(v)
    S = S0.clone()  # in place: state_out == state_in
    M = M0.clone() if beta else None
    a = _abi._seq_args(q, k, v, eta, None, beta, False, chunk, segments, S, M, o, S, M)
    need = int(L.ttt_la_workspace_size(ctypes.byref(a)))
    ws = torch.full((max(need, 16),), 0x7F, dtype=torch.uint8, device="cuda")  # stale-looking scratch
    a.workspace, a.workspace_bytes = ws.data_ptr(), need
    code = L.ttt_la_forward_chunked(ctypes.byref(a), st)
    assert code == 0, _abi.status_string(code)
    assert L.ttt_la_get_last_device_status(st) == _abi.OK
    assert L.ttt_la_debug_check_line(st) == 0
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, 1.0 / math.sqrt(d), beta, False, S0, M0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")
    if beta:
        assert_bf16(M, M_ref, "momentum")


# (d, B, H, T, wave tokens): the backward's reverse passes (chunk 128 for d = 64, 64 for d = 128)
BWD_CASES = [
    (64, 2, 3, 128 * 3 + 5, 0),    # look-back, a few segments per head
    (64, 1, 2, 128 * 20 + 3, 0),   # cooperative start states, one wave
    (128, 1, 2, 64 * 160 + 3, 64), # wave schedule, two waves
]


@pytest.mark.parametrize("d,B,H,T,wave_tokens", BWD_CASES)
def test_debug_build_backward_checks_stay_clean(d, B, H, T, wave_tokens, monkeypatch):
    from test_layers_causal_b200 import _abi
    if wave_tokens:
        monkeypatch.setenv("TTT_LA_WAVE_TOKENS", str(wave_tokens))
    L = _abi.debug_lib()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L.ttt_la_debug_check_line(st)
    L.ttt_la_get_last_device_status(st)
    q, k, v, eta = _inputs(B, H, T, d, 400 + d + T)
    g = torch.Generator().manual_seed(7)
    dO = torch.randn(v.shape, generator=g).to(torch.bfloat16).cuda()
    S0 = 0.1 * torch.randn(B, H, d, d, generator=g).cuda()
    dW = torch.randn(B, H, d, d, generator=g).cuda()
    a, out = _abi._chunked_grad_args(q, k, v, dO, eta, None, False, S0, dW)
    need = int(L.ttt_la_backward_chunked_workspace_size(ctypes.byref(a)))
    ws = torch.full((max(need, 16),), 0x7F, dtype=torch.uint8, device="cuda")
    a.workspace, a.workspace_bytes = ws.data_ptr(), need
    code = L.ttt_la_backward_chunked(ctypes.byref(a), st)
    assert code == 0, _abi.status_string(code)
    assert L.ttt_la_get_last_device_status(st) == _abi.OK
    assert L.ttt_la_debug_check_line(st) == 0
    ref = _abi.backward_recurrent(q, k, v, dO, eta, state_in=S0, grad_state=dW)
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dW0"):
        assert_bf16(out[n], f64(ref[n]), n)


@pytest.mark.parametrize("d,T", [(64, 64 * 5 + 3), (128, 64 * 3 + 1)])
def test_debug_build_momentum_backward_checks_stay_clean(d, T):
    """The chunkwise momentum backward (reverse and deta kernels) with every
    state given, ragged T, through the debug build."""
    from test_layers_causal_b200 import _abi
    L = _abi.debug_lib()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L.ttt_la_debug_check_line(st)
    L.ttt_la_get_last_device_status(st)
    q, k, v, eta = _inputs(2, 2, T, d, 500 + d + T)
    g = torch.Generator().manual_seed(9)
    dO = torch.randn(v.shape, generator=g).to(torch.bfloat16).cuda()
    S0, M0, dW, dM = (0.2 * torch.randn(2, 2, d, d, generator=g)).cuda(), (0.2 * torch.randn(2, 2, d, d, generator=g)).cuda(), \
        torch.randn(2, 2, d, d, generator=g).cuda(), torch.randn(2, 2, d, d, generator=g).cuda()
    a, out = _abi._chunked_grad_args(q, k, v, dO, eta, None, False, S0, dW, 0.9, M0, dM)
    need = int(L.ttt_la_backward_chunked_workspace_size(ctypes.byref(a)))
    ws = torch.full((max(need, 16),), 0x7F, dtype=torch.uint8, device="cuda")
    a.workspace, a.workspace_bytes = ws.data_ptr(), need
    code = L.ttt_la_backward_chunked(ctypes.byref(a), st)
    assert code == 0, _abi.status_string(code)
    assert L.ttt_la_get_last_device_status(st) == _abi.OK
    assert L.ttt_la_debug_check_line(st) == 0
    ref = _abi.backward_recurrent(q, k, v, dO, eta, beta=0.9, state_in=S0, mom_in=M0, grad_state=dW, grad_mom=dM)
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dW0", "dM0"):
        assert_bf16(out[n], f64(ref[n]), n)
