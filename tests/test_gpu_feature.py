"""GPU parity of the frozen-MLP feature map phi(x) = silu(W1 x) * (W3 x)
(ttt_la_feature_map) and of the layer built on it (feature map, then the
chunked forward) against the float64 oracle, on the same bf16 inputs.

Tolerance of the feature map, derived from its arithmetic: the kernel forms
W1 x and W3 x in fp32 from bf16 operands (error about d_in * 2^-24 of the
magnitudes), applies the gate in fp32 with the fast exponential and division
(relative error below 1e-5) and rounds the product to bf16 once (at most
2^-9 relative).  So every element must satisfy
    |phi - ref| <= 2^-8 |ref| + 1e-5 max|ref|,
twice the rounding bound plus a floor for the fp32 parts.  The layer on phi
keeps the bf16 tolerance of the chunked forward (2e-2 relative Frobenius).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import make_feature_weights, make_qkv
from tests.gpu_util import assert_bf16, f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from test_layers_causal_b200 import _abi

WIDTHS = [(64, 64), (64, 128), (128, 64), (128, 128)]


@pytest.fixture(autouse=True)
def _no_timed_out_wait():
    """Every test also requires that no in-kernel wait ran out."""
    yield
    assert _abi.device_status() == _abi.OK


def _x(B, H, T, d, seed):
    q, k, _, _ = make_qkv((B, H), T, d, d, seed, with_z=False)
    return q.to(torch.bfloat16).contiguous().cuda(), k.to(torch.bfloat16).contiguous().cuda()


def _weights(H, d_in, d_out, seed):
    W1, W3 = make_feature_weights(H, d_in, d_out, seed)
    return W1.cuda(), W3.cuda()


def _assert_phi(y, x, W1, W3, what):
    ref = oracle.feature_map_f64(f64(x), f64(W1), f64(W3))
    got = f64(y)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(ref))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of bound, worst excess " \
                          f"{float(np.max(np.abs(got - ref) - bound)):.3e}"
    assert_bf16(y, ref, what)


@pytest.mark.parametrize("d_in,d_out", WIDTHS)
def test_feature_map_two_inputs_ragged(d_in, d_out):
    B, H, T = 2, 3, 300  # 3 tiles per sequence, the last one 44 tokens
    q, k = _x(B, H, T, d_in, 11)
    W1, W3 = _weights(H, d_in, d_out, 12)
    # outputs inside guarded buffers: nothing may be written past T
    guard = torch.full((2, B * H * T * d_out + 4096), 7.0, device="cuda", dtype=torch.bfloat16)
    ys = [guard[i, :B * H * T * d_out].view(B, H, T, d_out) for i in range(2)]
    out = _abi.feature_map([q, k], W1, W3, out=ys)
    torch.cuda.synchronize()
    assert out[0].data_ptr() == ys[0].data_ptr()
    _assert_phi(out[0], q, W1, W3, "phi(q)")
    _assert_phi(out[1], k, W1, W3, "phi(k)")
    assert torch.all(guard[:, B * H * T * d_out:] == 7.0)


@pytest.mark.parametrize("T", [1, 127, 128, 129])
def test_feature_map_one_input_edges(T):
    B, H, d = 1, 2, 64
    q, _ = _x(B, H, T, d, 20 + T)
    W1, W3 = _weights(H, d, d, 21)
    (y,) = _abi.feature_map(q, W1, W3)
    torch.cuda.synchronize()
    _assert_phi(y, q, W1, W3, f"phi T={T}")


@pytest.mark.parametrize("H,B,T", [(64, 1, 300), (16, 3, 64), (5, 7, 1000)])
def test_feature_map_head_changes_inside_a_block(H, B, T):
    """Tile ranges that cross heads (and inputs) inside one block: the
    stacked weights are reloaded there."""
    q, k = _x(B, H, T, 128, 30 + H)
    W1, W3 = _weights(H, 128, 64, 31)
    yq, yk = _abi.feature_map([q, k], W1, W3)
    torch.cuda.synchronize()
    _assert_phi(yq, q, W1, W3, "phi(q)")
    _assert_phi(yk, k, W1, W3, "phi(k)")


@pytest.mark.parametrize("d_in,d_out", WIDTHS)
def test_feature_map_many_tiles_per_block(d_in, d_out):
    """About seven tiles per block (1024 tiles over the persistent grid): every
    TMEM accumulator and output buffer is reused several times."""
    B, H, T = 1, 8, 8192
    q, k = _x(B, H, T, d_in, 35)
    W1, W3 = _weights(H, d_in, d_out, 36)
    ys = [torch.full((B, H, T, d_out), float("nan"), device="cuda", dtype=torch.bfloat16) for _ in range(2)]
    yq, yk = _abi.feature_map([q, k], W1, W3, out=ys)
    torch.cuda.synchronize()
    _assert_phi(yq, q, W1, W3, "phi(q)")
    _assert_phi(yk, k, W1, W3, "phi(k)")


def test_feature_map_full_llm_shape():
    """B4 H16 T4096, d 64 -> 64, both inputs in one launch, every element."""
    B, H, T, d = 4, 16, 4096, 64
    q, k = _x(B, H, T, d, 41)
    W1, W3 = _weights(H, d, d, 42)
    yq, yk = _abi.feature_map([q, k], W1, W3)
    torch.cuda.synchronize()
    _assert_phi(yq, q, W1, W3, "phi(q)")
    _assert_phi(yk, k, W1, W3, "phi(k)")


def test_feature_map_extreme_preactivations():
    """Large positive and negative pre-activations: the gate saturates to
    the identity and to zero without overflow or NaN."""
    B, H, T, d = 1, 2, 256, 64
    q, _ = _x(B, H, T, d, 50)
    W1, W3 = _weights(H, d, d, 51)
    W1 = (W1.float() * 200.0).to(torch.bfloat16)  # pre-activations of order +-200
    (y,) = _abi.feature_map(q, W1, W3)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    _assert_phi(y, q, W1, W3, "phi saturated")


@pytest.mark.parametrize("d_in,d_out,beta,token_eta", [(64, 64, 0.0, True), (128, 128, 0.0, False),
                                                       (64, 128, 0.9, True), (128, 64, 0.9, False)])
def test_layer_on_phi_matches_oracle(d_in, d_out, beta, token_eta):
    B, H, T = 2, 2, 300
    q, k, v, z = make_qkv((B, H), T, d_in, d_out, 60)
    q, k, v = (x.to(torch.bfloat16).contiguous().cuda() for x in (q, k, v))
    eta = (torch.sigmoid(z) / math.sqrt(d_out)).float().cuda() if token_eta else None
    ec = 1.0 / math.sqrt(d_out)
    W1, W3 = _weights(H, d_in, d_out, 61)
    chunk = 128 if d_out == 128 else 64
    o, S, M = _abi.forward_chunked_phi(q, k, v, W1, W3, eta, eta_const=ec, beta=beta, chunk=chunk)
    torch.cuda.synchronize()
    o_ref, S_ref, M_ref = oracle.ttt_feature_layer_f64(f64(q), f64(k), f64(v), f64(eta) if token_eta else ec,
                                                       f64(W1), f64(W3), beta=beta)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "W_T")
    if beta:
        assert_bf16(M, M_ref, "M_T")


def test_unsupported_width_raises():
    q, _ = _x(1, 1, 64, 64, 70)
    W1, W3 = _weights(1, 64, 32, 71)
    with pytest.raises(_abi.TttError) as e:
        _abi.feature_map(q, W1, W3)
    assert e.value.code == _abi.ERR_UNSUPPORTED
