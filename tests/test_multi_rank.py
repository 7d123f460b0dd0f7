"""Multi-process (world size 2, gloo, CPU) checks of the multi-GPU plumbing:
the layer splits over independent sequences with no exchange on the data
path, and the timing reductions (barrier, max over ranks, whole-job
throughput) behave as the benchmark assumes."""
import os
import socket

import numpy as np
import pytest
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
