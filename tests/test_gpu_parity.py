"""GPU parity: every CUDA entry point against the float64 oracle on the same
seeded inputs, through the C ABI.  Sizes span several chunks and a ragged
last chunk; the full workloads are checked on sampled heads."""
import math

import pytest
import torch

from synth import CONFIGS, make_case, make_qkv
from tests.gpu_util import assert_bf16, assert_f32, oracle_forward

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import test_layers_causal_b200 as ttt


def _case(B, H, T, dk, dv, dtype, seed, token_eta=True, device="cuda"):
    q, k, v, z = make_qkv((B, H), T, dk, dv, seed)
    eta = (torch.sigmoid(z) / math.sqrt(dk)).float() if token_eta else None
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    q, k, v = (x.to(dt).contiguous() for x in (q, k, v))
    return (q.to(device), k.to(device), v.to(device), None if eta is None else eta.to(device),
            1.0 / math.sqrt(dk))


def _state(B, H, dv, dk, seed, scale=0.3):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(B, H, dv, dk, generator=g)).cuda()


# ------------------------------------------------------------- decode ----
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("beta,ascent", [(0.0, False), (0.9, False), (0.0, True), (0.5, True)])
def test_decode_step_parity(dtype, d, beta, ascent):
    N, H = 5, 3
    q, k, v, eta, ec = _case(N, H, 1, d, d, dtype, 20 + d)
    q, k, v, eta = q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous(), eta[:, :, 0].contiguous()
    S0 = _state(N, H, d, d, 1)
    M0 = _state(N, H, d, d, 2) if beta else None
    S, M = S0.clone(), (M0.clone() if M0 is not None else None)
    o = ttt.decode_step(q, k, v, S, M, eta=eta, beta=beta, ascent=ascent)
    o_ref, S_ref, M_ref = oracle_forward(q[:, :, None], k[:, :, None], v[:, :, None], eta[:, :, None], ec,
                                         beta, ascent, S0, M0)
    assert_f32(o.float(), o_ref[:, :, 0], "o") if dtype == "f32" else assert_bf16(o, o_ref[:, :, 0], "o", lead=1)
    assert_f32(S, S_ref, "state")
    if beta:
        assert_f32(M, M_ref, "momentum")


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_decode_step_past_2_31_state_elements(beta):
    """Maximum sizes for decode: the fp32 state of 4097 sequences x 32 heads x
    128 x 128 (2^31 + 2^19 elements, 8.6 GB; with momentum its buffer as
    large), updated in place by one bf16 step.  The first and the last
    (sequence, head), whose state offsets pass 2^31, are compared with the
    oracle's one-token recurrence from the same state."""
    N, H, d = 4097, 32, 128
    assert (N * H - 1) * d * d >= 2 ** 31
    g = torch.Generator(device="cuda").manual_seed(8)
    bf = torch.bfloat16
    q = (torch.randn(N, H, d, generator=g, device="cuda") / math.sqrt(d)).to(bf)
    k = (torch.randn(N, H, d, generator=g, device="cuda") / math.sqrt(d)).to(bf)
    v = torch.randn(N, H, d, generator=g, device="cuda").to(bf)
    eta = 0.1 * torch.rand(N, H, generator=g, device="cuda")
    S = torch.randn(N, H, d, d, generator=g, device="cuda").mul_(0.3)
    M = torch.randn(N, H, d, d, generator=g, device="cuda").mul_(0.3) if beta else None
    picks = [(0, 0), (N - 1, H - 1)]
    sls = {pk: (slice(pk[0], pk[0] + 1), slice(pk[1], pk[1] + 1)) for pk in picks}
    S0 = {pk: S[sl].clone() for pk, sl in sls.items()}
    M0 = {pk: (M[sl].clone() if beta else None) for pk, sl in sls.items()}
    o = ttt.decode_step(q, k, v, S, M, eta=eta, beta=beta)
    torch.cuda.synchronize()
    for pk, sl in sls.items():
        o_ref, S_ref, M_ref = oracle_forward(q[sl][:, :, None], k[sl][:, :, None], v[sl][:, :, None],
                                             eta[sl][:, :, None], 0.0, beta, False, S0[pk], M0[pk])
        assert_bf16(o[sl], o_ref[:, :, 0], f"o {pk}")
        assert_f32(S[sl], S_ref, f"state {pk}")
        if beta:
            assert_f32(M[sl], M_ref, f"momentum {pk}")
    del q, k, v, eta, S, M, o
    torch.cuda.empty_cache()


# ---------------------------------------------------------- recurrent ----
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_recurrent_parity(dtype, d, beta):
    B, H, T = 2, 2, 203
    q, k, v, eta, ec = _case(B, H, T, d, d, dtype, 30 + d)
    S0 = _state(B, H, d, d, 3)
    M0 = _state(B, H, d, d, 4) if beta else None
    o, S, M = ttt.forward_recurrent(q, k, v, eta, beta=beta, state_in=S0, mom_in=M0)
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, ec, beta, False, S0, M0)
    if dtype == "f32":
        assert_f32(o, o_ref, "o")
    else:
        assert_bf16(o, o_ref, "o")
    assert_f32(S, S_ref, "state") if dtype == "f32" else assert_bf16(S, S_ref, "state")
    if beta:
        assert_f32(M, M_ref, "momentum") if dtype == "f32" else assert_bf16(M, M_ref, "momentum")


def test_recurrent_ascent_and_const_eta():
    q, k, v, _, ec = _case(1, 3, 77, 64, 64, "f32", 5, token_eta=False)
    o, S, _ = ttt.forward_recurrent(q, k, v, None, eta_const=ec, ascent=True)
    o_ref, S_ref, _ = oracle_forward(q, k, v, None, ec, 0.0, True)
    assert_f32(o, o_ref, "o")
    assert_f32(S, S_ref, "state")


# ------------------------------------------------------ chunked, fp32 ----
def test_chunked_f32_tiny_config():
    c = CONFIGS["tiny_f32"]
    x = make_case(c)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, S, _ = ttt.forward_chunked(q, k, v, None, eta_const=x["eta_const"], chunk=c.chunk)
    o_ref, S_ref, _ = oracle_forward(q, k, v, None, x["eta_const"])
    assert_f32(o, o_ref, "o")
    assert_f32(S, S_ref, "state")


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("beta", [0.0, 0.9])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 48), (16, 64)])
def test_chunked_f32_parity(chunk, beta, dk, dv):
    B, H, T = 2, 2, 150
    q, k, v, eta, ec = _case(B, H, T, dk, dv, "f32", 40 + chunk)
    S0 = _state(B, H, dv, dk, 5)
    M0 = _state(B, H, dv, dk, 6) if beta else None
    o, S, M = ttt.forward_chunked(q, k, v, eta, beta=beta, chunk=chunk, state_in=S0, mom_in=M0, ascent=True)
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, ec, beta, True, S0, M0)
    assert_f32(o, o_ref, "o")
    assert_f32(S, S_ref, "state")
    if beta:
        assert_f32(M, M_ref, "momentum")


def test_chunked_f32_d128_no_momentum():
    q, k, v, eta, ec = _case(1, 2, 130, 128, 128, "f32", 9)
    o, S, _ = ttt.forward_chunked(q, k, v, eta, chunk=64)
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec)
    assert_f32(o, o_ref, "o")
    assert_f32(S, S_ref, "state")


# ------------------------------------------- chunked, bf16 tensor cores ----
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("chunk", [64, 128])
@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("token_eta", [True, False])
def test_chunked_tc_parity(d, chunk, segments, token_eta):
    B, H, T = 2, 3, 5 * chunk + 37  # several chunks and a ragged tail
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 50 + d + chunk, token_eta)
    S0 = _state(B, H, d, d, 7, scale=0.1)
    o, S, _ = ttt.forward_chunked(q, k, v, eta, eta_const=ec, chunk=chunk, segments=segments, state_in=S0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec, 0.0, False, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")


@pytest.mark.parametrize("d,chunk,segments", [(128, 64, 8), (128, 128, 6), (64, 64, 16)])
@pytest.mark.parametrize("with_state", [True, False])
def test_chunked_tc_many_segments(d, chunk, segments, with_state):
    """Enough segments that the start states come from the cooperative prefix
    (the look-back would read more than 192 KB of totals), ragged tail."""
    B, H, T = 1, 3, segments * 2 * chunk - 29
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 130 + d + segments)
    S0 = _state(B, H, d, d, 12, scale=0.1) if with_state else None
    o, S, _ = ttt.forward_chunked(q, k, v, eta, chunk=chunk, segments=segments, state_in=S0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec, 0.0, False, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")


@pytest.mark.parametrize("d,chunk,segments", [(128, 128, 6), (128, 64, 6), (64, 128, 14)])
@pytest.mark.parametrize("runs_of", [1, 2])
@pytest.mark.parametrize("token_eta", [True, False])
def test_chunked_tc_waves(d, chunk, segments, runs_of, token_eta, monkeypatch):
    """The wave schedule: several waves of `segments` runs of one or two chunks
    (ragged splits, a ragged last chunk), starting from W_0, including the
    wave-end state carried between waves and the final state of the last
    scan."""
    monkeypatch.setenv("TTT_LA_WAVE_TOKENS", str(runs_of * chunk))
    B, H, T = 1, 3, segments * 7 * chunk - 29
    plan = ttt.chunked_plan(B, H, T, d, d, chunk=chunk, segments=segments, eta=token_eta)
    assert plan["cooperative"] == 1 and plan["waves"] >= (3 if runs_of == 1 else 2), plan
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 140 + d + chunk + runs_of, token_eta)
    S0 = _state(B, H, d, d, 15, scale=0.1)
    o, S, _ = ttt.forward_chunked(q, k, v, eta, eta_const=ec, chunk=chunk, segments=segments, state_in=S0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec, 0.0, False, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")


@pytest.mark.parametrize("d,chunk,segments,waves", [(128, 128, 6, True), (128, 128, 3, False), (64, 64, 4, False)])
def test_chunked_tc_state_in_place(d, chunk, segments, waves, monkeypatch):
    """state_out may be state_in: W_T overwrites W_0 only after every block has
    read it (wave schedule over five waves, and decoupled look-back)."""
    monkeypatch.setenv("TTT_LA_WAVE_TOKENS", str(chunk))
    B, H, T = 1, 2, segments * 5 * chunk - 3
    plan = ttt.chunked_plan(B, H, T, d, d, chunk=chunk, segments=segments, eta=True)
    assert plan["cooperative"] == int(waves) and plan["waves"] == (5 if waves else 1)
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 160 + d + segments)
    S0 = _state(B, H, d, d, 16, scale=0.1)
    Sx = S0.clone()
    o, S, _ = ttt.forward_chunked(q, k, v, eta, chunk=chunk, segments=segments, state_in=Sx, state_out=Sx)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0 and S.data_ptr() == Sx.data_ptr()
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec, 0.0, False, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(Sx, S_ref, "state")


@pytest.mark.parametrize("H,segments", [(2, 3), (40, 2)])
def test_chunked_tc_momentum_state_in_place(H, segments):
    """With momentum, W_T and M_T may overwrite W_0 and M_0: cooperative
    prefix (H = 2, one wave) and decoupled look-back (H = 40: 80 blocks of
    one per SM would fit, so force a grid beyond one wave with d = 128 and
    B = 2)."""
    B, d, T = 2, 128, 64 * 7 + 5
    plan = ttt.chunked_plan(B, H, T, d, d, chunk=64, beta=0.9, segments=segments, eta=True)
    assert plan["cooperative"] == (1 if plan["blocks"] <= plan["resident"] else 0)
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 170 + H)
    S0 = _state(B, H, d, d, 17, scale=0.1)
    M0 = _state(B, H, d, d, 18, scale=0.1)
    Sx, Mx = S0.clone(), M0.clone()
    o, _, _ = ttt.forward_chunked(q, k, v, eta, beta=0.9, chunk=64, segments=segments, state_in=Sx, mom_in=Mx,
                                  state_out=Sx, mom_out=Mx)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, ec, 0.9, False, S0, M0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(Sx, S_ref, "state")
    assert_bf16(Mx, M_ref, "momentum")


@pytest.mark.parametrize("d,chunk", [(64, 64), (128, 128)])
def test_chunked_tc_ascent_zero_state_and_exact_multiple(d, chunk):
    B, H, T = 1, 2, 4 * chunk
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 60 + d, True)
    o, S, _ = ttt.forward_chunked(q, k, v, eta, chunk=chunk, ascent=True, segments=2)
    o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec, 0.0, True)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")


@pytest.mark.parametrize("d,chunk,segments,waves", [(64, 64, 3, False), (128, 128, 3, False), (128, 128, 6, True),
                                                    (128, 64, 6, True)])
@pytest.mark.parametrize("ascent", [False, True])
def test_chunked_tc_const_eta_fold(d, chunk, segments, waves, ascent, monkeypatch):
    """A constant learning rate runs with sigma * eta folded into P and the bf16
    copy of W (the state carried as W / (sigma * eta)): W_0 divided on entry,
    W_T multiplied on exit, in place, in the look-back and the wave schedule,
    descent and ascent."""
    monkeypatch.setenv("TTT_LA_WAVE_TOKENS", str(chunk))
    B, H, T = 1, 2, segments * 4 * chunk - 19
    plan = ttt.chunked_plan(B, H, T, d, d, chunk=chunk, segments=segments, eta=False)
    assert plan["cooperative"] == int(waves), plan
    q, k, v, _, _ = _case(B, H, T, d, d, "bf16", 180 + d + chunk + segments, token_eta=False)
    ec = 0.37 / math.sqrt(d)
    S0 = _state(B, H, d, d, 19, scale=0.2)
    Sx = S0.clone()
    o, S, _ = ttt.forward_chunked(q, k, v, None, eta_const=ec, chunk=chunk, segments=segments, ascent=ascent,
                                  state_in=Sx, state_out=Sx)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0 and S.data_ptr() == Sx.data_ptr()
    o_ref, S_ref, _ = oracle_forward(q, k, v, None, ec, 0.0, ascent, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(Sx, S_ref, "state")


@pytest.mark.parametrize("ec", [0.0, 1e-35])
def test_chunked_tc_const_eta_without_fold(ec):
    """eta = 0 and a scale below the fold's range run the K scaler as for a
    per-token rate: no update, o = W_0 q, W_T = W_0."""
    B, H, T, d = 1, 2, 3 * 128 + 5, 128
    q, k, v, _, _ = _case(B, H, T, d, d, "bf16", 190, token_eta=False)
    S0 = _state(B, H, d, d, 20, scale=0.2)
    o, S, _ = ttt.forward_chunked(q, k, v, None, eta_const=ec, chunk=128, segments=2, state_in=S0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, _ = oracle_forward(q, k, v, None, ec, 0.0, False, S0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")


def test_chunked_tc_short_sequences():
    """T shorter than a chunk, T = 1, and T one past a chunk boundary."""
    for T in (1, 17, 65):
        q, k, v, eta, ec = _case(2, 2, T, 64, 64, "bf16", 70 + T)
        o, S, _ = ttt.forward_chunked(q, k, v, eta, chunk=64)
        o_ref, S_ref, _ = oracle_forward(q, k, v, eta, ec)
        assert_bf16(o, o_ref, f"o T={T}")
        assert_bf16(S, S_ref, f"state T={T}")


def test_chunked_tc_query_is_key():
    q, k, v, eta, ec = _case(1, 2, 300, 128, 128, "bf16", 80)
    o, _, _ = ttt.forward_chunked(k, k, v, eta, chunk=128, segments=2)
    o_ref, _, _ = oracle_forward(k, k, v, eta, ec)
    assert_bf16(o, o_ref, "o")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("chunk", [64, 128])
@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("beta,ascent", [(0.9, False), (0.5, True)])
def test_chunked_tc_momentum_parity(d, chunk, segments, beta, ascent):
    B, H, T = 2, 2, 6 * 64 + 23
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 100 + d + chunk)
    S0 = _state(B, H, d, d, 8, scale=0.1)
    M0 = _state(B, H, d, d, 9, scale=0.1)
    o, S, M = ttt.forward_chunked(q, k, v, eta, beta=beta, ascent=ascent, chunk=chunk, segments=segments,
                                  state_in=S0, mom_in=M0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, ec, beta, ascent, S0, M0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")
    assert_bf16(M, M_ref, "momentum")


def _state_at_16_bytes(S):
    """The same values at an address that is 16- but not 32-byte aligned
    (the ABI promises callers only 16)."""
    flat = torch.empty(S.numel() + 4, device=S.device, dtype=S.dtype)
    out = flat[4:].view(S.shape)
    out.copy_(S)
    assert out.data_ptr() % 32 == 16
    return out


@pytest.mark.parametrize("beta,segments", [(0.0, 1), (0.0, 3), (0.9, 1), (0.9, 3)])
def test_chunked_tc_states_at_16_byte_alignment(beta, segments):
    B, H, T, d = 1, 2, 4 * 64 + 9, 128
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 120)
    S0 = _state_at_16_bytes(_state(B, H, d, d, 10, scale=0.1))
    M0 = _state_at_16_bytes(_state(B, H, d, d, 11, scale=0.1)) if beta else None
    o, S, M = ttt.forward_chunked(q, k, v, eta, beta=beta, chunk=64, segments=segments, state_in=S0, mom_in=M0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, ec, beta, False, S0, M0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")
    if beta:
        assert_bf16(M, M_ref, "momentum")


@pytest.mark.parametrize("d,segments,H", [(64, 12, 2), (128, 10, 2), (64, 12, 16), (128, 5, 32)])
def test_chunked_tc_momentum_many_segments(d, segments, H):
    """Start states with many segments.  A grid of at most one block per SM
    takes the cooperative prefix (H = 2); a larger grid the decoupled
    look-back, with inclusive states published beyond 8 segments (H = 16:
    192 blocks, 12 segments) and totals only below (H = 32: 160 blocks)."""
    B, T = 1, segments * 2 * 64 - 17
    q, k, v, eta, ec = _case(B, H, T, d, d, "bf16", 170 + d)
    S0 = _state(B, H, d, d, 13, scale=0.1)
    M0 = _state(B, H, d, d, 14, scale=0.1)
    o, S, M = ttt.forward_chunked(q, k, v, eta, beta=0.9, chunk=64, segments=segments, state_in=S0, mom_in=M0)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, eta, ec, 0.9, False, S0, M0)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")
    assert_bf16(M, M_ref, "momentum")


def test_chunked_tc_momentum_const_eta_zero_state():
    q, k, v, _, ec = _case(1, 3, 500, 128, 128, "bf16", 111, token_eta=False)
    o, S, M = ttt.forward_chunked(q, k, v, None, eta_const=ec, beta=0.9, chunk=128, segments=2)
    o_ref, S_ref, M_ref = oracle_forward(q, k, v, None, ec, 0.9)
    assert_bf16(o, o_ref, "o")
    assert_bf16(S, S_ref, "state")
    assert_bf16(M, M_ref, "momentum")


def test_chunked_segments_and_recurrent_agree():
    """Invariants on the GPU: the result does not depend on the segment split,
    and the chunked and recurrent paths compute the same layer."""
    q, k, v, eta, ec = _case(2, 2, 1000, 64, 64, "bf16", 90)
    o1, S1, _ = ttt.forward_chunked(q, k, v, eta, chunk=64, segments=1)
    o5, S5, _ = ttt.forward_chunked(q, k, v, eta, chunk=64, segments=5)
    orr, Sr, _ = ttt.forward_recurrent(q, k, v, eta)
    o1, o5, orr = o1.float(), o5.float(), orr.float()
    assert (o1 - o5).norm() / o1.norm() < 1e-2
    assert (S1 - S5).norm() / S1.norm() < 1e-2
    assert (o1 - orr).norm() / orr.norm() < 2e-2


# ------------------------------------------------ full-size workloads ----
def _full_case(name, heads):
    c = CONFIGS[name]
    x = make_case(c)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    eta = x["eta"].cuda() if x["eta"] is not None else None
    return c, x, q, k, v, eta, heads


@pytest.mark.parametrize("name,chunk,heads", [("llm_d64", 64, [(0, 0), (3, 15), (1, 7)]),
                                              ("long_d128", 128, [(0, 0), (0, 5)]),
                                              ("long_d128", 64, [(0, 2), (0, 7)]),
                                              ("momentum_d128", 128, [(0, 0), (1, 9)])])
def test_full_size_sampled_heads(name, chunk, heads):
    """The workloads at full size, in the launch configuration the benchmark
    times (automatic segments and schedule), on sampled heads against the
    oracle over the whole sequence."""
    c, x, q, k, v, eta, heads = _full_case(name, heads)
    o, S, M = ttt.forward_chunked(q, k, v, eta, eta_const=x["eta_const"], beta=c.beta, chunk=chunk)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    for b, h in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        o_ref, S_ref, M_ref = oracle_forward(q[sl], k[sl], v[sl], None if eta is None else eta[sl],
                                             x["eta_const"], c.beta)
        assert_bf16(o[sl], o_ref, f"o {name} head {b},{h}")
        assert_bf16(S[sl], S_ref, f"state {name} head {b},{h}")
        if c.beta:
            assert_bf16(M[sl], M_ref, f"momentum {name} head {b},{h}")


@pytest.mark.parametrize("chunk", [64, 128])
def test_long_context_schedules_agree(chunk):
    """Property at full size (all 8 heads): the benchmark's cooperative
    schedule and a single sequential pass per head (one segment) give the
    same layer."""
    c, x, q, k, v, eta, _ = _full_case("long_d128", [])
    plan = ttt.chunked_plan(c.B, c.H, c.T, c.d_k, c.d_v, chunk=chunk)
    assert plan["cooperative"] == 1
    o, S, _ = ttt.forward_chunked(q, k, v, None, eta_const=x["eta_const"], chunk=chunk)
    o_ref, S_ref, _ = ttt.forward_chunked(q, k, v, None, eta_const=x["eta_const"], chunk=chunk, segments=1)
    assert (o.float() - o_ref.float()).norm() / o_ref.float().norm() < 1e-2
    assert (S - S_ref).norm() / S_ref.norm() < 1e-2


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_chunked_tc_past_2_31_elements(beta):
    """Maximum sizes: q, k, v and o of 257 heads x 65536 tokens x d = 128
    (2^31 + 2^24 elements each, 4.3 GB in bf16), so the element offsets of the
    last heads pass 2^31.  Heads are independent: the first and the last head
    carry seeded inputs from the generator and are compared with the oracle
    over the whole sequence, the others hold seeded device noise of the same
    scale.  Both the automatic plan (one segment per head) and four segments
    per head (1028 blocks, decoupled look-back) are checked, without and
    with momentum."""
    H, T, d = 257, 65536, 128
    assert H * T * d > 2 ** 31
    qs, ks, vs, zs = make_qkv((1, 2), T, d, d, 31)
    eta_s = (torch.sigmoid(zs) / math.sqrt(d)).float()
    g = torch.Generator(device="cuda").manual_seed(5)
    bf = torch.bfloat16

    def noise():
        return (torch.randn(1, H, T, d, generator=g, device="cuda", dtype=bf) * (1.0 / math.sqrt(d))).to(bf)
    q, k, v = noise(), noise(), noise()
    eta = torch.full((1, H, T), 0.5 / math.sqrt(d), device="cuda")
    for j, h in enumerate((0, H - 1)):
        q[0, h], k[0, h], v[0, h] = qs[0, j].to(bf).cuda(), ks[0, j].to(bf).cuda(), vs[0, j].to(bf).cuda()
        eta[0, h] = eta_s[0, j].cuda()
    refs = {h: oracle_forward(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], eta[:, h:h + 1], 0.0, beta)
            for h in (0, H - 1)}
    for segments in (0, 4):
        o, S, M = ttt.forward_chunked(q, k, v, eta, beta=beta, chunk=128, segments=segments)
        torch.cuda.synchronize()
        assert ttt.device_status() == 0
        for h, (o_ref, S_ref, M_ref) in refs.items():
            assert_bf16(o[:, h:h + 1], o_ref, f"o head {h} segments {segments}")
            assert_bf16(S[:, h:h + 1], S_ref, f"state head {h} segments {segments}")
            if beta:
                assert_bf16(M[:, h:h + 1], M_ref, f"momentum head {h} segments {segments}")
        del o, S, M
    del q, k, v, eta
    torch.cuda.empty_cache()


@pytest.mark.parametrize("path", ["recurrent_bf16", "chunked_f32"])
def test_other_paths_past_2_31_elements(path):
    """Maximum sizes on the recurrent kernel (bf16) and the fp32 chunked
    kernel: 513 heads x 32768 tokens x d = 128 (2^31 + 2^22 elements per
    tensor).  The last head, whose element offsets pass 2^31, carries seeded
    inputs from the generator and is compared with the oracle over the whole
    sequence; the others hold seeded device noise of the same scale."""
    H, T, d = 513, 32768, 128
    assert (H - 1) * T * d >= 2 ** 31
    dt = torch.bfloat16 if path == "recurrent_bf16" else torch.float32
    qs, ks, vs, zs = make_qkv((1, 1), T, d, d, 51)
    eta_s = (torch.sigmoid(zs) / math.sqrt(d)).float()
    g = torch.Generator(device="cuda").manual_seed(7)

    def noise(scale):
        return (torch.randn(1, H, T, d, generator=g, device="cuda", dtype=dt) * scale).to(dt)
    q, k, v = noise(1.0 / math.sqrt(d)), noise(1.0 / math.sqrt(d)), noise(1.0)
    eta = torch.full((1, H, T), 0.5 / math.sqrt(d), device="cuda")
    h = H - 1
    q[0, h], k[0, h], v[0, h] = (t[0, 0].to(dt).cuda() for t in (qs, ks, vs))
    eta[0, h] = eta_s[0, 0].cuda()
    if path == "recurrent_bf16":
        o, S, _ = ttt.forward_recurrent(q, k, v, eta)
    else:
        o, S, _ = ttt.forward_chunked(q, k, v, eta, chunk=64)
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    sl = slice(h, h + 1)
    o_ref, S_ref, _ = oracle_forward(q[:, sl], k[:, sl], v[:, sl], eta[:, sl], 0.0)
    if dt == torch.float32:
        assert_f32(o[:, sl], o_ref, "o")
        assert_f32(S[:, sl], S_ref, "state")
    else:
        assert_bf16(o[:, sl], o_ref, "o")
        assert_bf16(S[:, sl], S_ref, "state")
    del q, k, v, eta, o, S
    torch.cuda.empty_cache()


# ------------------------------------------------ decode workload ----
def test_decode_workload_prefill_then_steps():
    """256 sequences x 16 heads, d = 128: chunked prefill of 2048 tokens, then
    512 decode steps.  Sampled sequences against the oracle over all 2560
    tokens; every head against one chunked pass over the 2560 tokens."""
    from synth import make_decode_inputs
    x = make_decode_inputs("cuda")
    pq, pk, pv = x["prefill"]
    sq, sk, sv = x["steps"]
    ec = x["eta_const"]
    N, H, T, d = pq.shape
    steps = sq.shape[0]
    _, S, _ = ttt.forward_chunked(pq, pk, pv, None, eta_const=ec, chunk=128)
    outs = torch.empty(steps, N, H, d, dtype=torch.bfloat16, device="cuda")
    for t in range(steps):
        ttt.decode_step(sq[t], sk[t], sv[t], S, eta_const=ec, out=outs[t])
    torch.cuda.synchronize()
    assert ttt.device_status() == 0
    # invariant over all heads: prefill + steps == one pass over the whole sequence
    fq = torch.cat([pq, sq.permute(1, 2, 0, 3)], dim=2).contiguous()
    fk = torch.cat([pk, sk.permute(1, 2, 0, 3)], dim=2).contiguous()
    fv = torch.cat([pv, sv.permute(1, 2, 0, 3)], dim=2).contiguous()
    del pq, pk, pv
    o_full, S_full, _ = ttt.forward_chunked(fq, fk, fv, None, eta_const=ec, chunk=128)
    o_dec = outs.permute(1, 2, 0, 3).float()
    o_tail = o_full[:, :, T:].float()
    assert float((o_dec - o_tail).norm() / o_tail.norm()) < 2e-2
    assert float((S - S_full).norm() / S_full.norm()) < 2e-2
    # oracle on sampled sequences (all heads), token by token over 2560 tokens
    for n in (0, N - 1):
        sl = slice(n, n + 1)
        o_ref, S_ref, _ = oracle_forward(fq[sl], fk[sl], fv[sl], None, ec)
        assert_bf16(o_dec[sl], o_ref[:, :, T:], f"decode outputs, sequence {n}")
        assert_bf16(S[sl], S_ref, f"state after decode, sequence {n}")


# ---------------------------------------------------- bounded waits ----
def test_wait_timeout_is_reported_not_hung():
    assert ttt.device_status() == 0
    ttt.selftest_wait_timeout(20_000_000)  # 20 ms on a barrier nothing completes
    assert ttt.device_status() == 4        # TTT_LA_ERR_TIMEOUT, read and cleared
    assert ttt.device_status() == 0
    # the context is still usable
    q, k, v, eta, ec = _case(1, 1, 64, 64, 64, "bf16", 3)
    o, _, _ = ttt.forward_chunked(q, k, v, eta, chunk=64)
    assert torch.isfinite(o.float()).all()
