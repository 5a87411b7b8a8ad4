"""Host-side model check of the mbarrier phase protocol of the tensor-core projection kernels
(no GPU).

`dtp_tc_kernel` (k-loop GEMM) and `dtp_fwd_kernel` (persistent forward) let one thread issue TMA
copies and tensor-core MMAs and wait on mbarriers by phase parity: a wait for the completion of
phase u (the u-th use of a barrier) tests parity u & 1, which only means "phase u is complete"
when the barrier has completed u or u + 1 phases at that moment -- with u - 1 completed the test
passes too early, with u + 2 it never passes.  The model below replays the kernels' issue and wait
sequences (stage and parity formulas as in the kernels) for many stage counts and lengths, with
the asynchronous completions (TMA transactions, tcgen05.commit arrivals, in order per barrier)
landing at adversarial times, and checks that every wait sees the barrier in {u, u+1} completed
phases, that the phase it waits for is really complete when it proceeds, and that a stage is only
refilled after the MMAs that read it completed.
"""
import random

import pytest


class Barrier:
    def __init__(self):
        self.issued = 0      # phases whose completion has been requested (commit / expect_tx)
        self.completed = 0   # phases completed

    def request(self):
        self.issued += 1

    def settle(self, rng, all_=False):
        """Complete some (or all) requested phases, in order."""
        if all_:
            self.completed = self.issued
        elif self.completed < self.issued:
            self.completed += rng.randint(0, self.issued - self.completed)

    def wait(self, u, rng, label):
        """Parity wait for phase u: legal only with u or u + 1 phases completed when it starts."""
        assert u <= self.completed + 1 and self.completed <= u + 1, \
            f"{label}: waiting for phase {u} with {self.completed} completed"
        assert u < self.issued, f"{label}: waits for phase {u} that nothing will complete"
        while self.completed <= u:     # the parity test fails until phase u completes
            self.settle(rng)
            if self.completed <= u and rng.random() < 0.5:
                self.settle(rng, all_=True)
        assert self.completed >= u + 1


def kloop(nk, stages, rng):
    """dtp_tc_kernel's thread 0: PF = STAGES - 2 tiles ahead; stage of tile t is t % STAGES."""
    pf = stages - 2
    full = [Barrier() for _ in range(stages)]
    free = [Barrier() for _ in range(stages)]
    done = Barrier()
    mma_done = set()                    # tiles whose MMAs are known complete
    loaded = {}                         # stage -> tile it holds

    def issue(t):
        st = t % stages
        if st in loaded:                # refilling: the MMAs of the tile it held must be done
            assert loaded[st] in mma_done, f"stage {st} refilled before tile {loaded[st]} was read"
        loaded[st] = t
        full[st].request()

    for t in range(min(pf, nk)):
        issue(t)
    for kt in range(nk):
        nx = kt + pf
        if nx < nk:
            st = nx % stages
            if nx >= stages:
                free[st].wait(nx // stages - 1, rng, "free")
                mma_done.add(nx - stages)
            issue(nx)
        s = kt % stages
        for b in full + free:
            b.settle(rng)
        full[s].wait(kt // stages, rng, "full")
        free[s].request()               # tcgen05.commit of tile kt's MMAs
    done.request()
    for b in free:
        b.settle(rng, all_=True)
    done.settle(rng, all_=True)
    done.wait(0, rng, "done")


def persistent_fwd(T, rng):
    """dtp_fwd_kernel's thread 0: two stages / accumulators, tile i in stage and accumulator i & 1."""
    full = [Barrier(), Barrier()]
    acc = [Barrier(), Barrier()]
    loaded = {}
    drained = set()

    def issue(i):
        s = i & 1
        if s in loaded:
            assert loaded[s] in drained or loaded[s] == i - 2, "stage refilled too early"
        loaded[s] = i
        full[s].request()

    if T > 0:
        issue(0)
    for i in range(T):
        s = i & 1
        if i >= 1:
            acc[s ^ 1].wait((i - 1) >> 1, rng, "acc")    # MMA(i-1) done: its stage and accumulator
            drained.add(i - 1)
        if i + 1 < T:
            issue(i + 1)
        for b in full + acc:
            b.settle(rng)
        full[s].wait(i >> 1, rng, "full")
        acc[s].request()                                  # commit of MMA(i)
    if T > 0:
        acc[(T - 1) & 1].wait((T - 1) >> 1, rng, "acc last")


@pytest.mark.parametrize("stages", [3, 4, 5, 6, 8])
def test_kloop_protocol(stages):
    rng = random.Random(stages)
    for nk in range(0, 26):
        for _ in range(20):
            kloop(nk, stages, rng)


def test_persistent_forward_protocol():
    rng = random.Random(7)
    for T in range(0, 30):
        for _ in range(20):
            persistent_fwd(T, rng)


def test_model_catches_wrong_phase_indices():
    """The check is not vacuous: a wait that lags two phases behind (its parity never matches
    again) and a wait one use ahead (for a phase nothing has requested yet) both trip it."""
    rng = random.Random(1)
    b = Barrier()
    for _ in range(3):
        b.request()
    b.settle(rng, all_=True)          # phases 0..2 completed
    with pytest.raises(AssertionError):
        b.wait(0, rng, "lagging")
    with pytest.raises(AssertionError):
        b.wait(3, rng, "ahead")
