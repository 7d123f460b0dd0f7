"""A model of the chunked tensor-core kernel's barrier protocol for the
128 x 128 tile with three phase-A slots (chunked_tc.cuh), checked on the CPU.

Every warp role is a generator of ("wait", barrier, use) and ("arrive",
barrier) events in the kernel's order: the TMA producer, the K scaler, the
MMA thread, the epilogue warps and the O store warp.  A wait on the u-th use
of a barrier needs u + 1 completed phases.  An mbarrier parity wait only
sees the parity of the barrier's current phase, so a wait that finds its
barrier two or more phases past the awaited one would block on the GPU: the
model flags it.  Random interleavings of the roles must neither deadlock nor
make such a wait, for every phase-A and phase-B chunk count up to a dozen,
in both start-state schedules (cooperative: the epilogue frees the score
columns as soon as it has read phase A's total; look-back: after the
inclusive state is out).
"""
import random

import pytest

NST = 2  # stages of the 128 x 128 tile


def _roles(nA, nB, mode):
    uses = lambda x: nA // 3 + (1 if x < nA % 3 else 0)  # noqa: E731  phase-A chunks in slot x

    def producer():
        for ia in range(nA):  # phase A: slot ia % 3
            x, u = ia % 3, ia // 3
            if u > 0:
                yield ("wait", f"emptyA{x}", u - 1)
            yield ("arrive", f"fullA{x}")
        for ib in range(nB):  # phase B: stage ib % 2; its first use waits for the slots on it
            s, u = ib % NST, ib // NST
            if u == 0:
                for x in (s, 2):
                    if uses(x) > 0:
                        yield ("wait", f"emptyA{x}", uses(x) - 1)
            else:
                yield ("wait", f"empty{s}", u - 1)
            yield ("arrive", f"full{s}")

    def scaler():
        for ia in range(nA):
            x, u = ia % 3, ia // 3
            yield ("wait", f"fullA{x}", u)
            yield ("arrive", f"kreadyA{x}")
        for ib in range(nB):
            s, u = ib % NST, ib // NST
            yield ("wait", f"full{s}", u)
            yield ("arrive", f"kready{s}")

    def mma():
        nread, pending = 0, False
        for ia in range(nA):
            x, u = ia % 3, ia // 3
            yield ("wait", f"kreadyA{x}", u)
            yield ("arrive", f"emptyA{x}")
            if ia == nA - 1:
                yield ("arrive", "adone")
                pending = True
        for itb in range(nB):
            s, u, b = itb % NST, itb // NST, itb & 1
            yield ("wait", f"kready{s}", u)
            if pending:  # the scores' columns hold phase A's total until it is read out
                yield ("wait", "a_read", nread)
                nread, pending = nread + 1, False
            yield ("arrive", "sc_full")
            yield ("wait", "wbf_ready", itb)
            if itb >= 2:
                yield ("wait", f"o_free{b}", (itb - 2) >> 1)
            yield ("arrive", "sdone")
            yield ("wait", "p_ready", itb)
            yield ("arrive", f"o_full{b}")

    def epilogue():
        if nA > 0:
            yield ("wait", "adone", 0)
            if mode == "coop":
                yield ("arrive", "a_read")
        if mode == "lookback" and nA > 0:
            yield ("arrive", "a_read")
        yield ("arrive", "wbf_ready")  # the start state
        for itb in range(nB):
            s, b = itb % NST, itb & 1
            yield ("wait", "sc_full", itb)
            yield ("wait", "sdone", itb)  # P overlays the Q/K slots
            yield ("arrive", "p_ready")
            if itb + 1 < nB:
                yield ("arrive", "wbf_ready")
            yield ("wait", f"o_full{b}", itb >> 1)
            yield ("arrive", f"o_free{b}")
            yield ("arrive", f"staged{s}")

    def store():
        for itb in range(nB):
            s = itb % NST
            yield ("wait", f"staged{s}", itb // NST)
            yield ("arrive", f"empty{s}")

    return [producer(), scaler(), mma(), epilogue(), store()]


def _run(nA, nB, mode, rng):
    roles = _roles(nA, nB, mode)
    done, cur, phases = [False] * len(roles), [None] * len(roles), {}
    while not all(done):
        progress = False
        order = list(range(len(roles)))
        rng.shuffle(order)
        for i in order:
            if done[i]:
                continue
            if cur[i] is None:
                try:
                    cur[i] = next(roles[i])
                except StopIteration:
                    done[i], progress = True, True
                    continue
            ev = cur[i]
            if ev[0] == "arrive":
                phases[ev[1]] = phases.get(ev[1], 0) + 1
                cur[i], progress = None, True
            elif phases.get(ev[1], 0) >= ev[2] + 1:
                assert phases[ev[1]] < ev[2] + 2, f"parity wait {ev} finds {phases[ev[1]]} phases done"
                cur[i], progress = None, True
        assert progress, f"deadlock: nA={nA} nB={nB} {mode}: {cur}"


@pytest.mark.parametrize("mode", ["coop", "lookback"])
def test_three_slot_phase_a_protocol(mode):
    rng = random.Random(7)
    for nA in range(0, 14):
        for nB in range(1, 12):
            for _ in range(8):
                _run(nA, nB, mode, rng)


def test_the_model_detects_a_missing_release():
    """A planted mistake: a producer that never waits for a phase-A slot to
    be released laps the slots (nine chunks through three slots).  The model
    must catch it in some interleaving: a parity wait that finds its barrier
    two phases on, or a deadlock."""
    def bad_roles(nA, nB):
        roles = _roles(nA, nB, "coop")

        def producer():  # never waits for emptyA: laps the phase-A slots
            for ia in range(nA):
                yield ("arrive", f"fullA{ia % 3}")
            for ib in range(nB):
                s, u = ib % NST, ib // NST
                if u > 0:
                    yield ("wait", f"empty{s}", u - 1)
                yield ("arrive", f"full{s}")
        roles[0] = producer()
        return roles
    rng = random.Random(1)
    failures = 0
    for _ in range(50):
        roles = bad_roles(9, 4)
        done, cur, phases = [False] * 5, [None] * 5, {}
        try:
            while not all(done):
                progress = False
                for i in rng.sample(range(5), 5):
                    if done[i]:
                        continue
                    if cur[i] is None:
                        try:
                            cur[i] = next(roles[i])
                        except StopIteration:
                            done[i], progress = True, True
                            continue
                    ev = cur[i]
                    if ev[0] == "arrive":
                        phases[ev[1]] = phases.get(ev[1], 0) + 1
                        cur[i], progress = None, True
                    elif phases.get(ev[1], 0) >= ev[2] + 1:
                        assert phases[ev[1]] < ev[2] + 2
                        cur[i], progress = None, True
                assert progress
        except AssertionError:
            failures += 1
    assert failures > 0
