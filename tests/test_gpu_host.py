"""GPU checks of the end-to-end entry point with host buffers
(ttt_la_forward_chunked_host): pieces of whole sequences copied in, run and
copied out on overlapping streams.  Compared with the float64 oracle and with
the device entry point on the same seeded inputs."""
import math

import pytest
import torch

from synth import make_qkv
from tests.gpu_util import assert_bf16, assert_f32, oracle_forward

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import test_layers_causal_b200 as ttt
    from test_layers_causal_b200 import _abi


def _host_case(B, H, T, d, dtype, seed, pinned=True):
    q, k, v, z = make_qkv((B, H), T, d, d, seed)
    eta = (torch.sigmoid(z) / math.sqrt(d)).float().contiguous()
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    q, k, v = (x.to(dt).contiguous() for x in (q, k, v))
    if pinned:
        q, k, v, eta = (x.pin_memory() for x in (q, k, v, eta))
    return q, k, v, eta


@pytest.mark.parametrize("B,H", [(3, 3), (1, 1), (4, 16)])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_path_matches_oracle_and_device_path(B, H, pinned):
    T, d = 333, 64
    q, k, v, eta = _host_case(B, H, T, d, "bf16", 140 + B * H, pinned)
    S0 = (0.1 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(5)))
    S_out = torch.empty(B, H, d, d)
    o, _ = _abi.forward_chunked_host(q, k, v, eta, chunk=64, state_in=S0, state_out=S_out)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    assert not o.is_cuda
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, 1.0 / math.sqrt(d), 0.0, False, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S_out, S_ref, "state")
    od, Sd, _ = ttt.forward_chunked(q.cuda(), k.cuda(), v.cuda(), eta.cuda(), chunk=64, state_in=S0.cuda())
    assert_bf16(o, od.cpu().double().numpy(), "o vs device path")


def test_host_path_momentum_and_f32():
    q, k, v, eta = _host_case(2, 3, 200, 128, "bf16", 150)
    S_out, M_out = torch.empty(2, 3, 128, 128), torch.empty(2, 3, 128, 128)
    o, _ = _abi.forward_chunked_host(q, k, v, eta, beta=0.9, chunk=64, state_out=S_out, mom_out=M_out)
    torch.cuda.synchronize()
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, 1.0 / math.sqrt(128), 0.9)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S_out, S_ref, "state")
    assert_bf16(M_out, M_ref, "momentum")
    q, k, v, eta = _host_case(1, 5, 150, 32, "f32", 151)
    o, _ = _abi.forward_chunked_host(q, k, v, eta, chunk=32)
    torch.cuda.synchronize()
    o_ref, _, _ = oracle_forward(q, k, v, eta, 1.0 / math.sqrt(32))
    assert_f32(o, o_ref, "o f32")


def test_host_path_reuses_staging_and_orders_on_the_stream():
    """Back-to-back calls on one staging buffer, with the inputs rewritten
    between them by the host after a synchronise, give each call's result."""
    q, k, v, eta = _host_case(2, 8, 256, 64, "bf16", 160)
    o1, st = _abi.forward_chunked_host(q, k, v, eta, chunk=64)
    torch.cuda.synchronize()
    first = o1.clone()
    q2, k2, v2, eta2 = _host_case(2, 8, 256, 64, "bf16", 161)
    o2, st2 = _abi.forward_chunked_host(q2, k2, v2, eta2, chunk=64, staging=st)
    assert st2 is st
    torch.cuda.synchronize()
    o_ref1, _, _ = oracle_forward(q, k, v, eta, 1.0 / 8)
    o_ref2, _, _ = oracle_forward(q2, k2, v2, eta2, 1.0 / 8)
    assert_bf16(first, o_ref1, "first call")
    assert_bf16(o2, o_ref2, "second call")
