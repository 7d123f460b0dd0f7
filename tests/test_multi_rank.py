"""Multi-process (world size 2, gloo, CPU) checks of the multi-GPU plumbing:
the layer splits over independent sequences with no exchange on the data
path, and the timing reductions (barrier, max over ranks, whole-job
throughput) behave as the benchmark assumes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))


def _timing_worker(rank, world, port, q):
    _env(rank, world, port)
    from test_layers_causal_b200 import ranks
    info = ranks.init(backend="gloo", timeout_s=60)
    ranks.barrier(info)
    mine = 10.0 + 5.0 * rank
    worst = ranks.max_over_ranks(mine, info)
    total = ranks.weak_scaling_tokens_per_s(16384, info.world, worst)
    q.put((rank, worst, total))
    ranks.finalize(info)


def _shard_worker(rank, world, port, outq):
    _env(rank, world, port)
    import torch
    import torch.distributed as dist

    import oracle
    from synth import make_qkv
    from test_layers_causal_b200 import ranks
    info = ranks.init(backend="gloo", timeout_s=60)
    B, H, T, d = 5, 2, 37, 8
    q, k, v, z = make_qkv((B, H), T, d, d, seed=31)  # every rank draws the same global batch
    eta = torch.sigmoid(z) / d ** 0.5
    sl = ranks.local_slice(B, info.rank, info.world)
    f = lambda t: t.double().numpy()  # noqa: E731
    o_local, W_local, _ = oracle.ttt_recurrence_f64(f(q[sl]), f(k[sl]), f(v[sl]), f(eta[sl]), beta=0.9)
    # gather only to check the result; the layer itself exchanges nothing
    parts = [None] * info.world
    dist.all_gather_object(parts, (sl.start, sl.stop, o_local, W_local))
    if info.rank == 0:
        o_full, W_full, _ = oracle.ttt_recurrence_f64(f(q), f(k), f(v), f(eta), beta=0.9)
        covered = np.zeros(B, dtype=int)
        for a, b, o_p, W_p in parts:
            covered[a:b] += 1
            assert np.array_equal(o_p, o_full[a:b]) and np.array_equal(W_p, W_full[a:b])
        outq.put(("ok", covered.tolist()))
    ranks.finalize(info)


def _oracle_backend():
    """The three operations of the sequence split computed by the float64
    oracle, so the orchestration (slicing, all-gather, which maps compose
    where) runs on CPU ranks.  The map's scalars come from the recurrence
    itself: G from how M_0 = 1 enters W, B from how it decays."""
    import oracle
    from test_layers_causal_b200.seqshard import Backend

    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731

    def seg_map(q, k, v, eta, eta_const=None, beta=0.0, ascent=False, chunk=64):
        e = f(eta) if eta is not None else eta_const
        _, W, M = oracle.ttt_recurrence_f64(f(q), f(k), f(v), e, beta=beta, ascent=ascent)
        if not beta:
            return torch.from_numpy(W), None, None
        ones = np.ones_like(W)
        _, W1, M1 = oracle.ttt_recurrence_f64(f(q), f(k), f(v), e, beta=beta, ascent=ascent, M0=ones)
        G = -(W1 - W).mean(axis=(-2, -1))
        B = (M1 - M).mean(axis=(-2, -1))
        return torch.from_numpy(W), torch.from_numpy(M), torch.from_numpy(np.stack([G, B], -1))

    def compose(dW, dM, GB, W0, M0):
        w = f(W0) if W0 is not None else np.zeros(dW.shape[1:])
        m = f(M0) if M0 is not None else np.zeros(dW.shape[1:])
        for j in range(dW.shape[0]):
            G = f(GB[j])[..., 0, None, None] if GB is not None else 0.0
            B = f(GB[j])[..., 1, None, None] if GB is not None else 1.0
            w = w - G * m + f(dW[j])
            m = B * m + f(dM[j]) if dM is not None else m
        return torch.from_numpy(w), torch.from_numpy(m)

    def forward(q, k, v, eta, state_in=None, mom_in=None, return_state=False, eta_const=None, beta=0.0,
                ascent=False, chunk=64):
        e = f(eta) if eta is not None else eta_const
        o, W, M = oracle.ttt_recurrence_f64(f(q), f(k), f(v), e, beta=beta, ascent=ascent, S0=f(state_in),
                                            M0=f(mom_in))
        return torch.from_numpy(o), torch.from_numpy(W), torch.from_numpy(M)

    def backward(q, k, v, dO, eta, eta_const=None, beta=0.0, ascent=False, state_in=None, mom_in=None,
                 grad_state=None, grad_mom=None):
        e = f(eta) if eta is not None else eta_const
        r = oracle.ttt_backward_f64(f(q), f(k), f(v), e, f(dO), f(grad_state), f(grad_mom), beta=beta,
                                    ascent=ascent, S0=f(state_in), M0=f(mom_in))
        return {n: torch.from_numpy(np.ascontiguousarray(x)) for n, x in r.items()}

    return Backend(segment_map=seg_map, compose_maps=compose, forward=forward, backward=backward)


def _seqshard_worker(rank, world, port, outq):
    _env(rank, world, port)
    import torch.distributed as dist

    import oracle
    from synth import make_qkv
    from test_layers_causal_b200 import ranks, seqshard
    info = ranks.init(backend="gloo", timeout_s=60)
    B, H, T, d = 2, 2, 53, 6
    q, k, v, z = make_qkv((B, H), T, d, d, seed=41)  # every rank draws the whole sequence
    eta = torch.sigmoid(z) / d ** 0.5
    g = torch.Generator().manual_seed(3)
    S0, M0 = 0.2 * torch.randn(B, H, d, d, generator=g), 0.2 * torch.randn(B, H, d, d, generator=g)
    res = {}
    for beta in (0.0, 0.9):
        sl = seqshard.token_slice(T, info.rank, info.world)
        loc = lambda x: x[:, :, sl].contiguous()  # noqa: E731
        o, W_T, M_T = seqshard.forward_sequence_sharded(
            loc(q), loc(k), loc(v), loc(eta), rank=info.rank, world=info.world, beta=beta,
            state_in=S0.double(), mom_in=M0.double() if beta else None, backend=_oracle_backend())
        parts = [None] * info.world
        dist.all_gather_object(parts, (sl.start, sl.stop, o.numpy(), W_T.numpy(),
                                       None if M_T is None else M_T.numpy()))
        f = lambda t: t.double().numpy()  # noqa: E731
        o_ref, W_ref, M_ref = oracle.ttt_recurrence_f64(f(q), f(k), f(v), f(eta), beta=beta, S0=f(S0),
                                                        M0=f(M0) if beta else None)
        err = 0.0
        covered = np.zeros(T, dtype=int)
        for a, b, o_p, W_p, M_p in parts:
            covered[a:b] += 1
            err = max(err, np.abs(o_p - o_ref[:, :, a:b]).max(), np.abs(W_p - W_ref).max())
            if beta:
                err = max(err, np.abs(M_p - M_ref).max())
        res[beta] = (err, covered.tolist())
    if info.rank == 0:
        outq.put(res)
    ranks.finalize(info)


def _seqshard_bwd_worker(rank, world, port, outq):
    _env(rank, world, port)
    import torch.distributed as dist

    import oracle
    from synth import make_qkv
    from test_layers_causal_b200 import ranks, seqshard
    info = ranks.init(backend="gloo", timeout_s=60)
    B, H, T, d = 2, 2, 47, 5
    q, k, v, z = make_qkv((B, H), T, d, d, seed=43)  # every rank draws the whole sequence
    eta = torch.sigmoid(z) / d ** 0.5
    g = torch.Generator().manual_seed(4)
    S0, M0, dW_T, dM_T = (0.2 * torch.randn(B, H, d, d, generator=g) for _ in range(4))
    dO = torch.randn(B, H, T, d, generator=g)
    sl = seqshard.token_slice(T, info.rank, info.world)
    loc = lambda x: x[:, :, sl].contiguous()  # noqa: E731
    f = lambda t: t.double().numpy()  # noqa: E731
    res = {}
    for beta, ascent in ((0.0, False), (0.0, True), (0.8, False), (0.6, True)):
        mom = dict(mom_in=M0.double(), grad_mom=dM_T.double()) if beta else {}
        dq, dk, dv, deta, dW0, dM0 = seqshard.backward_sequence_sharded(
            loc(q), loc(k), loc(v), loc(dO), loc(eta), rank=info.rank, world=info.world, beta=beta, ascent=ascent,
            state_in=S0.double(), grad_state=dW_T.double(), backend=_oracle_backend(), **mom)
        parts = [None] * info.world
        dist.all_gather_object(parts, (sl.start, sl.stop, dq.numpy(), dk.numpy(), dv.numpy(), deta.numpy(),
                                       dW0.numpy(), None if dM0 is None else dM0.numpy()))
        ref = oracle.ttt_backward_f64(f(q), f(k), f(v), f(eta), f(dO), f(dW_T), f(dM_T) if beta else None,
                                      beta=beta, ascent=ascent, S0=f(S0), M0=f(M0) if beta else None)
        err = 0.0
        covered = np.zeros(T, dtype=int)
        for a, b, dq_p, dk_p, dv_p, de_p, dW0_p, dM0_p in parts:
            covered[a:b] += 1
            err = max(err, np.abs(dq_p - ref["dq"][:, :, a:b]).max(), np.abs(dk_p - ref["dk"][:, :, a:b]).max(),
                      np.abs(dv_p - ref["dv"][:, :, a:b]).max(), np.abs(de_p - ref["deta"][:, :, a:b]).max(),
                      np.abs(dW0_p - ref["dW0"]).max())
            if beta:
                err = max(err, np.abs(dM0_p - ref["dM0"]).max())
        res[(beta, ascent)] = (err, covered.tolist())
    if info.rank == 0:
        outq.put(res)
    ranks.finalize(info)


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("rank did not finish")
        assert p.exitcode == 0
    out = []
    while not q.empty():
        out.append(q.get())
    return out


def test_timing_reduction_two_ranks():
    out = sorted(_run(_timing_worker))
    assert [r for r, _, _ in out] == [0, 1]
    for _, worst, total in out:
        assert worst == 15.0                       # slowest rank's time on every rank
        assert abs(total - 16384 * 2 / 15e-3) < 1  # all ranks' tokens over that time


def test_sequences_shard_with_no_exchange():
    out = _run(_shard_worker)
    assert out == [("ok", [1, 1, 1, 1, 1])]       # every sequence owned by exactly one rank


@pytest.mark.parametrize("B,world", [(4, 2), (5, 2), (3, 4), (1, 8), (16, 8)])
def test_local_slice_partitions_the_batch(B, world):
    from test_layers_causal_b200 import ranks
    seen = []
    for r in range(world):
        sl = ranks.local_slice(B, r, world)
        seen.extend(range(B)[sl])
    assert seen == list(range(B))


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_split_over_ranks_matches_the_whole_sequence(world):
    """Two or three CPU ranks each hold a contiguous run of every sequence;
    after the all-gather of the runs' maps and the composition, every run's
    output and the final (W, M) equal the whole-sequence recurrence."""
    (res,) = _run(_seqshard_worker, world=world)
    for beta, (err, covered) in res.items():
        assert covered == [1] * 53, beta
        assert err < 1e-12, (beta, err)


@pytest.mark.parametrize("world", [2, 3])
def test_backward_sequence_split_over_ranks_matches_the_whole_sequence(world):
    """The backward over two or three CPU ranks, with and without momentum:
    each rank's dq, dk, dv, deta for its run and the common dL/dW_0, dL/dM_0
    equal the whole-sequence gradient oracle (one all-gather of the forward
    maps, one of the runs' constant terms, the later runs' adjoint maps
    folded onto the final-state gradients)."""
    (res,) = _run(_seqshard_bwd_worker, world=world)
    for key, (err, covered) in res.items():
        assert covered == [1] * 47, key
        assert err < 1e-11, (key, err)


def test_library_backward_takes_the_chunked_form_where_it_exists():
    """seqshard.LIBRARY runs a run's backward chunk-parallel for the shapes
    ttt_la_backward_chunked takes, and recurrent otherwise (host logic only)."""
    import torch
    from test_layers_causal_b200.seqshard import chunked_backward_supported as ok
    bf, f32 = torch.bfloat16, torch.float32
    t = lambda d, dt: torch.empty(1, 1, 4, d, dtype=dt)  # noqa: E731
    assert ok(t(64, bf), t(64, bf), 0.0) and ok(t(128, bf), t(128, bf), 0.9)
    assert not ok(t(32, bf), t(32, bf), 0.0) and not ok(t(64, bf), t(128, bf), 0.0)
    assert ok(t(48, f32), t(64, f32), 0.0) and not ok(t(48, f32), t(64, f32), 0.9)
    assert not ok(t(130, f32), t(64, f32), 0.0) and not ok(t(30, f32), t(64, f32), 0.0)
