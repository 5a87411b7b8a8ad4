"""Host-side model check of the mbarrier phase protocol of the tensor-core projection kernels
(no GPU).

`dtp_tc_kernel` (k-loop GEMM) runs a copy thread and an MMA thread concurrently;
`dtp_fwd_ws_kernel` (persistent forward) a copy thread, an MMA thread and four drain warps.  They
wait on mbarriers by phase parity: a wait for the completion of
phase u (the u-th use of a barrier) tests parity u & 1, which only means "phase u is complete"
when the barrier has completed u or u + 1 phases at that moment -- with u - 1 completed the test
passes too early, with u + 2 it never passes.  The model below replays the kernels' issue and wait
sequences (stage and parity formulas as in the kernels) for many stage counts and lengths, with
the asynchronous completions (TMA transactions, tcgen05.commit arrivals, in order per barrier)
landing at adversarial times (and, for the warp-specialised kernel, the roles interleaved at
random), and checks that every wait sees the barrier in {u, u+1} completed phases, that the phase
it waits for is really complete when it proceeds, that a stage is only refilled after the MMAs
that read it completed, and that an accumulator is only overwritten after every drain warp read
it.
"""
import random

import pytest


class CBarrier:
    """An mbarrier of the concurrent model: `count` arrivals complete a phase (arrive); or an
    asynchronous completion requested now lands later, in order (request / settle)."""

    def __init__(self, count=1):
        self.count, self.arrived, self.completed, self.issued = count, 0, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived = 0
            self.completed += 1

    def request(self):
        self.issued += 1

    def settle(self, rng):
        if self.completed < self.issued and rng.random() < 0.5:
            self.completed += 1

    def wait(self, u, label):
        """Generator: a parity wait for phase u, polling until phase u is complete; every poll
        must see u or u + 1 completed phases (else the parity test would pass early or never)."""
        while True:
            assert self.completed in (u, u + 1), f"{label}: phase {u} polled with {self.completed} completed"
            if self.completed == u + 1:
                return
            yield


def ws_forward(units, stages, acc, rng):
    """dtp_fwd_ws_kernel: copy thread, MMA thread and four drain warps, interleaved at random.
    `units` lists the output tiles of each unit (one u tile in A buffer k % 2, then that many w
    tiles through the stage ring)."""
    afull = [CBarrier() for _ in range(2)]
    afree = [CBarrier() for _ in range(2)]
    full = [CBarrier() for _ in range(stages)]
    freeb = [CBarrier() for _ in range(stages)]
    accf = [CBarrier() for _ in range(acc)]
    acce = [CBarrier(4) for _ in range(acc)]
    asyncs = afull + afree + full + freeb + accf
    T = sum(units)
    abuf_unit, units_done = {}, set()
    stage_tile, acc_tile, mma_done, drained = {}, {}, set(), {}

    def producer():
        i = 0
        for k, nj in enumerate(units):
            ab = k & 1
            if k >= 2:
                yield from afree[ab].wait((k >> 1) - 1, "A free")
                assert abuf_unit[ab] in units_done, f"A buffer {ab} refilled before unit {abuf_unit[ab]} was done"
            abuf_unit[ab] = k
            afull[ab].request()
            for _ in range(nj):
                s, r = i % stages, i // stages
                if r >= 1:
                    yield from freeb[s].wait(r - 1, "free")
                    assert stage_tile[s] in mma_done, f"stage {s} refilled before tile {stage_tile[s]} was read"
                stage_tile[s] = i
                full[s].request()
                i += 1
                yield

    def mma():
        i = 0
        for k, nj in enumerate(units):
            ab = k & 1
            yield from afull[ab].wait(k >> 1, "A full")
            assert abuf_unit[ab] == k, f"unit {k} multiplied from an A buffer holding {abuf_unit[ab]}"
            for _ in range(nj):
                s, ac = i % stages, i % acc
                yield from full[s].wait(i // stages, "full")
                assert stage_tile[s] == i, f"tile {i} multiplied from a stage holding {stage_tile[s]}"
                if i >= acc:
                    yield from acce[ac].wait(i // acc - 1, "acc free")
                    assert drained.get(i - acc, 0) == 4, f"accumulator of tile {i - acc} overwritten early"
                acc_tile[ac] = i
                mma_done.add(i)        # the commits below land only after the MMAs completed
                freeb[s].request()
                accf[ac].request()
                i += 1
                yield
            units_done.add(k)
            afree[ab].request()

    def drain(w):
        for i in range(T):
            ac = i % acc
            yield from accf[ac].wait(i // acc, f"acc full (warp {w})")
            assert acc_tile[ac] == i, f"warp {w} drained tile {acc_tile[ac]} for {i}"
            drained[i] = drained.get(i, 0) + 1
            acce[ac].arrive()
            yield

    actors = [producer(), mma()] + [drain(w) for w in range(4)]
    while actors:
        for b in asyncs:
            b.settle(rng)
        a = rng.choice(actors)
        try:
            next(a)
        except StopIteration:
            actors.remove(a)
    assert all(drained.get(i, 0) == 4 for i in range(T))


@pytest.mark.parametrize("stages,acc", [(2, 4), (3, 4), (4, 4), (2, 2), (3, 2), (4, 3)])
def test_warp_specialised_forward_protocol(stages, acc):
    rng = random.Random(stages * 10 + acc)
    for n in range(0, 9):
        for _ in range(15):
            ws_forward([rng.randint(1, 5) for _ in range(n)], stages, acc, rng)


def ws_kloop(nk, stages, rng):
    """dtp_tc_kernel: copy thread (tile t into stage t % STAGES) and MMA thread, interleaved."""
    full = [CBarrier() for _ in range(stages)]
    freeb = [CBarrier() for _ in range(stages)]
    done = CBarrier()
    stage_tile, mma_done = {}, set()

    def producer():
        for t in range(nk):
            st = t % stages
            if t >= stages:
                yield from freeb[st].wait(t // stages - 1, "free")
                assert stage_tile[st] in mma_done, f"stage {st} refilled before tile {stage_tile[st]} was read"
            stage_tile[st] = t
            full[st].request()
            yield

    def mma():
        for kt in range(nk):
            s = kt % stages
            yield from full[s].wait(kt // stages, "full")
            assert stage_tile[s] == kt, f"tile {kt} multiplied from a stage holding {stage_tile[s]}"
            mma_done.add(kt)
            freeb[s].request()
            yield
        done.request()
        yield from done.wait(0, "done")

    actors = [producer(), mma()]
    while actors:
        for b in full + freeb + [done]:
            b.settle(rng)
        a = rng.choice(actors)
        try:
            next(a)
        except StopIteration:
            actors.remove(a)
    assert mma_done == set(range(nk))


@pytest.mark.parametrize("stages", [2, 3, 4, 5, 6, 8])
def test_kloop_protocol(stages):
    rng = random.Random(stages)
    for nk in range(0, 26):
        for _ in range(20):
            ws_kloop(nk, stages, rng)


def test_model_catches_wrong_phase_indices():
    """The check is not vacuous: a wait that lags two phases behind (its parity never matches
    again) and a wait two phases ahead (its parity would pass at once) both trip it."""
    b = CBarrier()
    for _ in range(3):
        b.arrive()                    # phases 0..2 completed
    with pytest.raises(AssertionError):
        next(b.wait(0, "lagging"))
    with pytest.raises(AssertionError):
        next(b.wait(4, "ahead"))
