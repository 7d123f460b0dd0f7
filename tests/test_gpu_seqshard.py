"""GPU checks of the sequence split along T: each run's affine map
(ttt_la_segment_map), the composition of maps (ttt_la_compose_maps) and the
forward from a composed start state reproduce the float64 oracle run over
the whole sequence.  The ranks are simulated one after the other on one GPU;
the exchange itself is covered on CPU ranks in test_multi_rank.py."""
import math

import pytest
import torch

import oracle
from synth import make_qkv
from tests.gpu_util import assert_bf16, assert_f32, f64, oracle_forward

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from test_layers_causal_b200 import _abi, seqshard


def _inputs(B, H, T, d, dtype, seed, token_eta=True):
    q, k, v, z = make_qkv((B, H), T, d, d, seed)
    eta = (torch.sigmoid(z) / math.sqrt(d)).float().cuda() if token_eta else None
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    return (*(x.to(dt).contiguous().cuda() for x in (q, k, v)), eta)


@pytest.mark.parametrize("beta,ascent,token_eta", [(0.0, False, True), (0.9, False, True), (0.5, True, False),
                                                   (0.0, True, False)])
@pytest.mark.parametrize("world", [2, 3])
def test_runs_compose_to_the_whole_sequence(beta, ascent, token_eta, world):
    B, H, T, d = 2, 2, 3 * 64 * 2 + 41, 64
    q, k, v, eta = _inputs(B, H, T, d, "bf16", 190 + world, token_eta)
    ec = 1.0 / math.sqrt(d)
    g = torch.Generator().manual_seed(21)
    S0 = (0.1 * torch.randn(B, H, d, d, generator=g)).cuda()
    M0 = (0.1 * torch.randn(B, H, d, d, generator=g)).cuda() if beta else None
    kw = dict(eta_const=ec, beta=beta, ascent=ascent, chunk=64)
    sl = [seqshard.token_slice(T, r, world) for r in range(world)]
    run = lambda x, s: None if x is None else x[:, :, s].contiguous()  # noqa: E731
    maps = [_abi.segment_map(run(q, s), run(k, s), run(v, s), run(eta, s), **kw) for s in sl]
    dW = torch.stack([m[0] for m in maps])
    dM = torch.stack([m[1] for m in maps]) if beta else None
    GB = torch.stack([m[2] for m in maps]) if beta else None
    outs = []
    for r, s in enumerate(sl):
        W0, M0r = _abi.compose_maps(dW[:r], None if dM is None else dM[:r], None if GB is None else GB[:r], S0, M0)
        o, _, _ = _abi.forward_chunked(run(q, s), run(k, s), run(v, s), run(eta, s), state_in=W0,
                                       mom_in=M0r if beta else None, return_state=False, **kw)
        outs.append(o)
    W_T, M_T = _abi.compose_maps(dW, dM, GB, S0, M0)
    torch.cuda.synchronize()
    o_ref, W_ref, M_ref = oracle_forward(q, k, v, eta, ec, beta, ascent, S0, M0)
    assert_bf16(torch.cat(outs, dim=2), o_ref, "o")
    assert_bf16(W_T, W_ref, "W_T")
    if beta:
        assert_bf16(M_T, M_ref, "M_T")


def test_compose_is_exact_elementwise_and_module_world_one():
    """compose_maps against the map formula on random maps (fp32 both sides,
    same operation order), and the module at world size 1 (no exchange)."""
    g = torch.Generator().manual_seed(5)
    n, B, H, d = 3, 2, 3, 32
    dW, dM = (torch.randn(n, B, H, d, d, generator=g).cuda() for _ in range(2))
    GB = torch.rand(n, B, H, 2, generator=g).cuda()
    W0, M0 = (torch.randn(B, H, d, d, generator=g).cuda() for _ in range(2))
    W, M = _abi.compose_maps(dW, dM, GB, W0, M0)
    w, m = W0.clone(), M0.clone()
    for j in range(n):
        G_, B_ = GB[j, ..., 0, None, None], GB[j, ..., 1, None, None]
        w = torch.addcmul(w, -G_.expand_as(m), m) + dW[j]
        m = torch.addcmul(dM[j], B_.expand_as(m), m)
    assert_f32(W, w.cpu().double().numpy(), "W")
    assert_f32(M, m.cpu().double().numpy(), "M")
    q, k, v, eta = _inputs(1, 2, 200, 64, "bf16", 99)
    o, W_T, _ = seqshard.forward_sequence_sharded(q, k, v, eta, chunk=64)
    o_ref, W_ref, _ = oracle_forward(q, k, v, eta, 1.0 / 8)
    assert_bf16(o, o_ref, "o")
    assert_bf16(W_T, W_ref, "W_T")


@pytest.mark.parametrize("form", ["recurrent", "chunked"])
@pytest.mark.parametrize("world", [1, 2, 3])
def test_backward_runs_compose_to_the_whole_sequence(world, form):
    """The backward split without momentum, ranks one after another: each run's
    start state from the forward maps, its own do q^T sum from a backward with
    no final-state gradient, the later runs' sums added onto dL/dW_T, then the
    run's backward; dq, dk, dv, deta of every run and dL/dW_0 against the
    whole-sequence gradient oracle, with the runs' backward in either form."""
    bwd = _abi.backward_recurrent if form == "recurrent" else _abi.backward_chunked
    B, H, T, d = 2, 2, 3 * 32 + 17, 64
    x = _inputs(B, H, T, d, "bf16", 210 + world)
    q, k, v, eta = x
    g = torch.Generator().manual_seed(22)
    S0 = (0.1 * torch.randn(B, H, d, d, generator=g)).cuda()
    dW_T = torch.randn(B, H, d, d, generator=g).cuda()
    dO = torch.randn(B, H, T, d, generator=g).to(torch.bfloat16).cuda()
    ec = 1.0 / math.sqrt(d)
    sl = [seqshard.token_slice(T, r, world) for r in range(world)]
    run = lambda t, s: t[:, :, s].contiguous()  # noqa: E731
    maps = torch.stack([_abi.segment_map(run(q, s), run(k, s), run(v, s), run(eta, s), eta_const=ec, chunk=64)[0]
                        for s in sl])
    starts = [_abi.compose_maps(maps[:r], None, None, S0, None)[0] for r in range(world)]
    own = torch.stack([bwd(run(q, s), run(k, s), run(v, s), run(dO, s), run(eta, s), eta_const=ec,
                           state_in=starts[r])["dW0"] for r, s in enumerate(sl)])
    parts = []
    for r, s in enumerate(sl):
        G_end, _ = _abi.compose_maps(own[r + 1:], None, None, dW_T, None)
        parts.append(bwd(run(q, s), run(k, s), run(v, s), run(dO, s), run(eta, s), eta_const=ec,
                         state_in=starts[r], grad_state=G_end))
    dW0, _ = _abi.compose_maps(own, None, None, dW_T, None)
    torch.cuda.synchronize()
    ref = oracle.ttt_backward_f64(f64(q), f64(k), f64(v), f64(eta), f64(dO), f64(dW_T), S0=f64(S0))
    for n in ("dq", "dk", "dv", "deta"):
        assert_bf16(torch.cat([p[n] for p in parts], dim=2), ref[n], n)
    assert_bf16(dW0, ref["dW0"], "dW0")
    if world == 1 and form == "chunked":  # the module itself (its runs take the chunked form), no exchange
        dq, dk, dv, deta, dW0m, dM0m = seqshard.backward_sequence_sharded(q, k, v, dO, eta, eta_const=ec,
                                                                          state_in=S0, grad_state=dW_T)
        assert dM0m is None
        torch.cuda.synchronize()
        assert_bf16(dq, ref["dq"], "module dq")
        assert_bf16(dW0m, ref["dW0"], "module dW0")


def test_backward_module_with_momentum_world_one():
    """backward_sequence_sharded with momentum on one rank: the adjoint fold
    of its own run (ttt_la_compose_maps with per-head scalars) gives dL/dM_0,
    and the run's gradients equal the whole-sequence oracle."""
    B, H, T, d = 2, 2, 2 * 64 + 9, 64
    q, k, v, eta = _inputs(B, H, T, d, "bf16", 230)
    g = torch.Generator().manual_seed(23)
    S0, M0 = ((0.1 * torch.randn(B, H, d, d, generator=g)).cuda() for _ in range(2))
    dW_T, dM_T = (torch.randn(B, H, d, d, generator=g).cuda() for _ in range(2))
    dO = torch.randn(B, H, T, d, generator=g).to(torch.bfloat16).cuda()
    ec = 1.0 / math.sqrt(d)
    dq, dk, dv, deta, dW0, dM0 = seqshard.backward_sequence_sharded(
        q, k, v, dO, eta, eta_const=ec, beta=0.9, state_in=S0, mom_in=M0, grad_state=dW_T, grad_mom=dM_T)
    torch.cuda.synchronize()
    ref = oracle.ttt_backward_f64(f64(q), f64(k), f64(v), f64(eta), f64(dO), f64(dW_T), f64(dM_T), beta=0.9,
                                  S0=f64(S0), M0=f64(M0))
    for n, x in (("dq", dq), ("dk", dk), ("dv", dv), ("deta", deta), ("dW0", dW0), ("dM0", dM0)):
        assert_bf16(x, ref[n], n)
