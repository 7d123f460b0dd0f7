"""GPU parity of the layer's backward (ttt_la_backward_recurrent) against the
float64 gradient oracle on the same inputs.

Tolerances as for the forward: fp32 inputs, max |x - ref| / max |ref| <= 1e-4
per gradient; bf16 inputs (fp32 arithmetic, gradients rounded to bf16),
relative Frobenius error <= 2e-2 per (b, h) slice and overall.  Sizes span
several 32-token checkpoint chunks and a ragged last one.
"""
import math

import pytest
import torch

import oracle
from synth import make_qkv
from tests.gpu_util import assert_bf16, assert_f32, f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from test_layers_causal_b200 import _abi


@pytest.fixture(autouse=True)
def _no_timed_out_wait():
    yield
    assert _abi.device_status() == _abi.OK


def _case(B, H, T, dk, dv, dtype, seed, token_eta=True, states=True):
    q, k, v, z = make_qkv((B, H), T, dk, dv, seed)
    g = torch.Generator().manual_seed(seed + 1000)
    dO = torch.randn(B, H, T, dv, generator=g)
    S0 = 0.3 * torch.randn(B, H, dv, dk, generator=g) if states else None
    M0 = 0.3 * torch.randn(B, H, dv, dk, generator=g) if states else None
    dW = torch.randn(B, H, dv, dk, generator=g) if states else None
    dM = torch.randn(B, H, dv, dk, generator=g) if states else None
    eta = (torch.sigmoid(z) / math.sqrt(dk)).float() if token_eta else None
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    dev = lambda x: None if x is None else x.contiguous().cuda()  # noqa: E731
    return dict(q=dev(q.to(dt)), k=dev(k.to(dt)), v=dev(v.to(dt)), dO=dev(dO.to(dt)), eta=dev(eta), S0=dev(S0),
                M0=dev(M0), dW=dev(dW), dM=dev(dM), ec=1.0 / math.sqrt(dk))


def _run(x, beta, ascent):
    return _abi.backward_recurrent(x["q"], x["k"], x["v"], x["dO"], x["eta"], eta_const=x["ec"], beta=beta,
                                   ascent=ascent, state_in=x["S0"], mom_in=x["M0"] if beta else None,
                                   grad_state=x["dW"], grad_mom=x["dM"] if beta else None)


def _ref(x, beta, ascent):
    e = f64(x["eta"]) if x["eta"] is not None else x["ec"]
    return oracle.ttt_backward_f64(f64(x["q"]), f64(x["k"]), f64(x["v"]), e, f64(x["dO"]), f64(x["dW"]),
                                   f64(x["dM"]) if beta else None, beta=beta, ascent=ascent, S0=f64(x["S0"]),
                                   M0=f64(x["M0"]) if beta else None)


@pytest.mark.parametrize("beta,ascent", [(0.0, False), (0.0, True), (0.9, False), (0.5, True)])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 48), (128, 128)])
def test_backward_f32_matches_oracle(beta, ascent, dk, dv):
    x = _case(2, 2, 100, dk, dv, "f32", 7 + dk)
    got = _run(x, beta, ascent)
    torch.cuda.synchronize()
    ref = _ref(x, beta, ascent)
    for n in ("dq", "dk", "dv", "deta", "dW0") + (("dM0",) if beta else ()):
        assert_f32(got[n], ref[n], n)


@pytest.mark.parametrize("beta", [0.0, 0.9])
@pytest.mark.parametrize("dk", [64, 128])
def test_backward_bf16_matches_oracle(beta, dk):
    x = _case(2, 3, 257, dk, dk, "bf16", 31 + dk, token_eta=(beta == 0.0))
    got = _run(x, beta, False)
    torch.cuda.synchronize()
    ref = _ref(x, beta, False)
    for n in ("dq", "dk", "dv", "deta", "dW0") + (("dM0",) if beta else ()):
        assert_bf16(got[n], ref[n], n)


@pytest.mark.parametrize("T", [1, 31, 32, 33])
def test_backward_short_sequences_without_states(T):
    x = _case(1, 2, T, 64, 64, "f32", 50 + T, states=False)
    got = _run(x, 0.9, False)
    torch.cuda.synchronize()
    ref = _ref(x, 0.9, False)
    for n in ("dq", "dk", "dv", "deta", "dW0", "dM0"):
        assert_f32(got[n], ref[n], n)


def test_backward_is_the_gradient_of_the_gpu_forward():
    """Directional check through the library alone: for a small step along a
    random direction, the change of <o, dO> computed by the GPU forward
    (fp32 recurrent) matches the GPU gradient's inner product with that
    direction."""
    x = _case(1, 2, 64, 32, 32, "f32", 77, states=False)
    g = _run(x, 0.0, False)
    gen = torch.Generator().manual_seed(78)
    dirs = {n: torch.randn(x[n].shape, generator=gen).cuda() for n in ("q", "k", "v")}
    h = 1e-3

    def L(sign):
        o, _, _ = _abi.forward_recurrent(*(x[n] + sign * h * dirs[n] for n in ("q", "k", "v")), x["eta"],
                                         eta_const=x["ec"])
        return float((o.double() * x["dO"].double()).sum())

    fd = (L(1) - L(-1)) / (2 * h)
    an = sum(float((g["d" + n].double() * dirs[n].double()).sum()) for n in ("q", "k", "v"))
    assert abs(fd - an) <= 1e-3 * max(1.0, abs(an)), (fd, an)
