"""GPU parity of the chunk-parallel backward without momentum
(ttt_la_backward_chunked: three runs of the chunked forward) against the
float64 gradient oracle and against the recurrent backward.

Tolerances: bf16 inputs, relative Frobenius error <= 2e-2 per (b, h) slice
and overall; fp32 inputs (the fp32 chunked forward), max-rel <= 1e-4.
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
    g = torch.Generator().manual_seed(seed + 2000)
    dO = torch.randn(B, H, T, dv, generator=g)
    S0 = 0.3 * torch.randn(B, H, dv, dk, generator=g) if states else None
    dW = torch.randn(B, H, dv, dk, generator=g) if states else None
    eta = (torch.sigmoid(z) / math.sqrt(dk)).float() if token_eta else None
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    dev = lambda x: None if x is None else x.contiguous().cuda()  # noqa: E731
    return dict(q=dev(q.to(dt)), k=dev(k.to(dt)), v=dev(v.to(dt)), dO=dev(dO.to(dt)), eta=dev(eta), S0=dev(S0),
                dW=dev(dW), ec=1.0 / math.sqrt(dk))


def _ref(x, ascent):
    e = f64(x["eta"]) if x["eta"] is not None else x["ec"]
    return oracle.ttt_backward_f64(f64(x["q"]), f64(x["k"]), f64(x["v"]), e, f64(x["dO"]), f64(x["dW"]),
                                   ascent=ascent, S0=f64(x["S0"]))


@pytest.mark.parametrize("d,T,token_eta,ascent,states", [(64, 300, True, False, True), (128, 257, False, True, True),
                                                         (64, 64, True, False, False), (128, 1, True, False, True),
                                                         (64, 100, True, True, True), (128, 33, True, False, False)])
def test_backward_chunked_bf16_matches_oracle(d, T, token_eta, ascent, states):
    x = _case(2, 3, T, d, d, "bf16", 90 + d + T, token_eta, states)
    g = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], eta_const=x["ec"], ascent=ascent,
                              state_in=x["S0"], grad_state=x["dW"])
    torch.cuda.synchronize()
    ref = _ref(x, ascent)
    for n in ("dq", "dk", "dv", "deta", "dW0"):
        assert_bf16(g[n], ref[n], n)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 48)])
def test_backward_chunked_f32_matches_oracle(dk, dv):
    x = _case(2, 2, 150, dk, dv, "f32", 120 + dk + dv)
    g = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], eta_const=x["ec"], state_in=x["S0"],
                              grad_state=x["dW"])
    torch.cuda.synchronize()
    ref = _ref(x, False)
    for n in ("dq", "dk", "dv", "deta", "dW0"):
        assert_f32(g[n], ref[n], n)


def test_backward_chunked_agrees_with_recurrent_at_llm_shape():
    """B4 H16 T4096 d64, per-token eta: the two backward forms agree."""
    x = _case(4, 16, 4096, 64, 64, "bf16", 140)
    a = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], state_in=x["S0"], grad_state=x["dW"])
    b = _abi.backward_recurrent(x["q"], x["k"], x["v"], x["dO"], x["eta"], state_in=x["S0"], grad_state=x["dW"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dW0"):
        assert_bf16(a[n], f64(b[n]), n)


@pytest.mark.parametrize("d,T,wave_tokens", [(128, 64 * 400 + 5, 0), (128, 64 * 400 + 5, 128),
                                             (64, 128 * 150 + 3, 0), (64, 128 * 150 + 3, 256)])
def test_backward_chunked_long_sequence_schedules(d, T, wave_tokens, monkeypatch):
    """Two heads of a long ragged sequence: the reverse passes run tens of
    segments per head with the cooperative start states, in one wave or
    (TTT_LA_WAVE_TOKENS) in several, and agree with the recurrent backward."""
    if wave_tokens:
        monkeypatch.setenv("TTT_LA_WAVE_TOKENS", str(wave_tokens))
    x = _case(1, 2, T, d, d, "bf16", 170 + d)
    a = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], ascent=True, state_in=x["S0"],
                              grad_state=x["dW"])
    b = _abi.backward_recurrent(x["q"], x["k"], x["v"], x["dO"], x["eta"], ascent=True, state_in=x["S0"],
                                grad_state=x["dW"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dW0"):
        assert_bf16(a[n], f64(b[n]), n)


def _mom_case(B, H, T, d, seed, token_eta=True, states=True):
    x = _case(B, H, T, d, d, "bf16", seed, token_eta, states)
    g = torch.Generator().manual_seed(seed + 3000)
    x["M0"] = (0.3 * torch.randn(B, H, d, d, generator=g)).cuda() if states else None
    x["dM"] = torch.randn(B, H, d, d, generator=g).cuda() if states else None
    return x


@pytest.mark.parametrize("d,T,token_eta,ascent,states", [(64, 300, True, False, True), (128, 257, True, True, True),
                                                         (64, 1, True, True, True), (128, 64, False, False, False),
                                                         (128, 1, True, False, True), (64, 129, False, True, True)])
def test_backward_chunked_momentum_matches_oracle(d, T, token_eta, ascent, states):
    """beta = 0.9: dq from the momentum forward, dv / dk / dW0 / dM0 from the
    reverse chunkwise kernel, deta from the forward-order one."""
    x = _mom_case(2, 3, T, d, 210 + d + T, token_eta, states)
    g = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], eta_const=x["ec"], ascent=ascent,
                              state_in=x["S0"], grad_state=x["dW"], beta=0.9, mom_in=x["M0"], grad_mom=x["dM"])
    torch.cuda.synchronize()
    e = f64(x["eta"]) if x["eta"] is not None else x["ec"]
    ref = oracle.ttt_backward_f64(f64(x["q"]), f64(x["k"]), f64(x["v"]), e, f64(x["dO"]), f64(x["dW"]),
                                  f64(x["dM"]), beta=0.9, ascent=ascent, S0=f64(x["S0"]), M0=f64(x["M0"]))
    for n in ("dq", "dk", "dv", "deta", "dW0", "dM0"):
        assert_bf16(g[n], ref[n], n)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_chunked_momentum_agrees_with_recurrent(d):
    """Four heads of a long ragged sequence (dozens of chunks carried by one
    block each): the chunkwise and recurrent momentum backwards agree."""
    x = _mom_case(1, 4, 64 * 60 + 7, d, 260 + d)
    kw = dict(state_in=x["S0"], grad_state=x["dW"], beta=0.9, mom_in=x["M0"], grad_mom=x["dM"], ascent=True)
    a = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], **kw)
    b = _abi.backward_recurrent(x["q"], x["k"], x["v"], x["dO"], x["eta"], **kw)
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dW0", "dM0"):
        assert_bf16(a[n], f64(b[n]), n)


def test_backward_chunked_momentum_two_streams_and_graph_capture():
    """With momentum the call runs its three independent launch chains on
    three streams. The outputs are the same bits on the default stream, on
    another stream, and replayed from a captured CUDA graph, which the side
    streams join through the call's fork and join events."""
    x = _mom_case(2, 3, 64 * 9 + 5, 128, 280)
    kw = dict(eta_const=x["ec"], state_in=x["S0"], grad_state=x["dW"], beta=0.9, mom_in=x["M0"], grad_mom=x["dM"])
    a = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], **kw)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], **kw)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        c = _abi.backward_chunked(x["q"], x["k"], x["v"], x["dO"], x["eta"], **kw)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dW0", "dM0"):
        assert torch.equal(a[n], b[n]), n
        assert torch.equal(a[n], c[n]), n


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_backward_chunked_past_2_31_elements(beta):
    """Maximum sizes: q, k, v, dO and the gradients of 513 heads x 32768
    tokens x d = 128 (2^31 + 2^22 elements each, 4.3 GB in bf16).  Heads are
    independent: the last head, whose element offsets pass 2^31, carries
    seeded inputs from the generator and is compared with the gradient
    oracle; the others hold seeded device noise of the same scale."""
    H, T, d = 513, 32768, 128
    assert (H - 1) * T * d >= 2 ** 31
    qs, ks, vs, zs = make_qkv((1, 1), T, d, d, 41)
    dOs = torch.randn(1, 1, T, d, generator=torch.Generator().manual_seed(42))
    eta_s = (torch.sigmoid(zs) / math.sqrt(d)).float()
    g = torch.Generator(device="cuda").manual_seed(6)
    bf = torch.bfloat16

    def noise(scale):
        return (torch.randn(1, H, T, d, generator=g, device="cuda", dtype=bf) * scale).to(bf)
    q, k, v, dO = noise(1.0 / math.sqrt(d)), noise(1.0 / math.sqrt(d)), noise(1.0), noise(1.0)
    eta = torch.full((1, H, T), 0.5 / math.sqrt(d), device="cuda")
    h = H - 1
    q[0, h], k[0, h], v[0, h], dO[0, h] = (t[0, 0].to(bf).cuda() for t in (qs, ks, vs, dOs))
    eta[0, h] = eta_s[0, 0].cuda()
    gr = _abi.backward_chunked(q, k, v, dO, eta, beta=beta)
    torch.cuda.synchronize()
    sl = slice(h, h + 1)
    ref = oracle.ttt_backward_f64(f64(q[:, sl]), f64(k[:, sl]), f64(v[:, sl]), f64(eta[:, sl]), f64(dO[:, sl]), None,
                                  beta=beta)
    for n in ("dq", "dk", "dv", "deta", "dW0") + (("dM0",) if beta else ()):
        assert_bf16(gr[n][:, sl], ref[n], f"{n} head {h}")
    del q, k, v, dO, eta, gr
    torch.cuda.empty_cache()
