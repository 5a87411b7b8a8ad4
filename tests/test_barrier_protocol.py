"""Host-side model check of the named-barrier hand-over in the warp-specialised kernels (no GPU).

The Flash PD-SSM backward (`pdssm_bwd_kernel`: a scan warp and a score warp per pair) and the
complex-mode forward, backward (from the trajectory and from checkpoints) and RTRL kernels
(`cplx_*_kernel`: four producer warps and two consumer warps per CTA) hand two shared buffers over
with bar.sync / bar.arrive on FULL and EMPTY barriers.  A barrier completes a phase when the warps of its count have arrived (bar.arrive) or
are waiting (bar.sync); a warp must not arrive twice in one phase.  The sequences below are the
kernels' barrier operations in program order, per role; the simulation runs them for 0 to 12
tiles and checks that every role finishes (no deadlock), that no role contributes twice to one
phase, and that every barrier ends with no partial phase.  A second model replays the
checkpointed backward's copy schedule (which tiles each item's copies bring, and when).
"""

import pytest


def simulate(programs, weights, counts):
    """programs: role -> list of (op, barrier); weights: role -> warps; counts: barrier -> warps."""
    pc = {r: 0 for r in programs}
    waiting = {}                                   # role -> barrier it is blocked on
    arrived = {b: 0 for b in counts}               # warps in the current phase
    members = {b: set() for b in counts}           # roles in the current phase
    blocked_in = {b: set() for b in counts}

    def complete(b):
        arrived[b] = 0
        members[b] = set()
        for r in blocked_in[b]:
            waiting.pop(r, None)
        blocked_in[b] = set()

    progress = True
    while progress:
        progress = False
        for r, prog in programs.items():
            if r in waiting or pc[r] >= len(prog):
                continue
            op, b = prog[pc[r]]
            assert r not in members[b], f"{r} joins phase of barrier {b} twice"
            members[b].add(r)
            arrived[b] += weights[r]
            assert arrived[b] <= counts[b], f"barrier {b} over-subscribed"
            pc[r] += 1
            progress = True
            if arrived[b] == counts[b]:
                complete(b)
            elif op == "sync":
                waiting[r] = b
                blocked_in[b].add(r)
    stuck = {r: programs[r][pc[r] - 1] for r in waiting}
    assert not stuck, f"deadlock: {stuck}"
    assert all(pc[r] == len(p) for r, p in programs.items())
    assert all(v == 0 for v in arrived.values()), f"partial phases left: {arrived}"


FULL, EMPTY = (1, 2), (3, 4)


def pd_bwd(ntiles):
    scan = [op for i in range(ntiles) for op in (("sync", EMPTY[i & 1]), ("arrive", FULL[i & 1]))]
    scan += [("sync", EMPTY[0]), ("sync", EMPTY[1])]
    score = [("arrive", EMPTY[0]), ("arrive", EMPTY[1])]
    score += [op for i in range(ntiles) for op in (("sync", FULL[i & 1]), ("arrive", EMPTY[i & 1]))]
    return {"scan": scan, "score": score}, {"scan": 1, "score": 1}, {b: 2 for b in FULL + EMPTY}


PROD, CONS = 5, 6


def cplx(ntiles, kind):
    if kind == "fwd":
        prod = [op for i in range(ntiles)
                for op in (("sync", PROD), ("sync", EMPTY[i & 1]), ("arrive", FULL[i & 1]))]
    else:  # bwd, rtrl: the step scalars are written after EMPTY
        prod = [op for i in range(ntiles)
                for op in (("sync", EMPTY[i & 1]), ("sync", PROD), ("arrive", FULL[i & 1]))]
    prod += [("sync", EMPTY[0]), ("sync", EMPTY[1])]
    tail = (("sync", CONS),) if kind == "bwd" else ()  # the column sums after the sweep
    cons = [("arrive", EMPTY[0]), ("arrive", EMPTY[1])]
    cons += [op for i in range(ntiles)
             for op in (("sync", CONS), ("sync", FULL[i & 1]), ("arrive", EMPTY[i & 1])) + tail]
    counts = {b: 6 for b in FULL + EMPTY}
    counts[PROD], counts[CONS] = 4, 2
    return {"prod": prod, "cons": cons}, {"prod": 4, "cons": 2}, counts


@pytest.mark.parametrize("ntiles", range(13))
def test_pdssm_backward_hand_over(ntiles):
    simulate(*pd_bwd(ntiles))


@pytest.mark.parametrize("kind", ["fwd", "bwd", "rtrl"])
@pytest.mark.parametrize("ntiles", range(13))
def test_complex_hand_over(kind, ntiles):
    simulate(*cplx(ntiles, kind))


def test_a_missing_release_is_caught():
    progs, w, c = pd_bwd(3)
    progs["scan"] = progs["scan"][:-1]  # drop the scan warp's last balancing sync
    with pytest.raises(AssertionError):
        simulate(progs, w, c)
    progs, w, c = pd_bwd(3)
    progs["score"] = progs["score"][1:]  # the score warp forgets to pre-release buffer 0
    with pytest.raises(AssertionError):
        simulate(progs, w, c)


def ckpt_items(nts):
    """Item sequence of the checkpointed complex backward for chunks of nts[0], nts[1], ... tiles
    (in processing order): each chunk's tiles forward, then the same tiles as sweep items in
    reverse, as (chunk, sweep, tile, tiles of the chunk)."""
    items = []
    for c, nt in enumerate(nts):
        items += [(c, False, j, nt) for j in range(nt)]
        items += [(c, True, j, nt) for j in reversed(range(nt))]
    return items


def cplx_ckpt(nts):
    items = ckpt_items(nts)
    prod = [op for i in range(len(items))
            for op in (("sync", EMPTY[i & 1]), ("sync", PROD), ("arrive", FULL[i & 1]))]
    prod += [("sync", EMPTY[0]), ("sync", EMPTY[1])]
    cons = [("arrive", EMPTY[0]), ("arrive", EMPTY[1])]
    for i, (_, sweep, j, nt) in enumerate(items):
        cons += [("sync", CONS), ("sync", FULL[i & 1]), ("arrive", EMPTY[i & 1])]
        if sweep or j == nt - 1:  # the column sums, or the chunk's h_{t-1} all written
            cons.append(("sync", CONS))
    counts = {b: 6 for b in FULL + EMPTY}
    counts[PROD], counts[CONS] = 4, 2
    return {"prod": prod, "cons": cons}, {"prod": 4, "cons": 2}, counts


CKPT_CHUNKS = [[], [1], [3], [8], [2, 8], [8, 8, 8], [5, 8, 8, 8]]


@pytest.mark.parametrize("nts", CKPT_CHUNKS)
def test_complex_checkpointed_hand_over(nts):
    simulate(*cplx_ckpt(nts))


def ckpt_copy_schedule(nts, defer=True):
    """Replays the consumers' copies in `cplx_bwd_ckpt_kernel`: item i + 1's u or g tile is
    issued at the start of item i, and a sweep item's h_{t-1} rows too, except (defer) for a
    chunk's first sweep item, whose rows are issued after the barrier that ends the chunk's last
    forward item.  Asserts that every item's tiles are issued before it waits for its copies,
    that every h_{t-1} row is copied only after the forward item that writes it has finished, and
    that no copy lands in the stage the current item reads."""
    items = ckpt_items(nts)
    issued = {0: {"x"}}          # prologue: item 0 (a forward item) needs only its u tile
    done_fwd = set()             # (chunk, tile) whose forward item has finished
    for i, (chunk, sweep, j, nt) in enumerate(items):
        need = {"x", "h"} if sweep else {"x"}
        assert need <= issued.get(i, set()), f"item {i} waits for copies never issued"
        late = defer and not sweep and j == nt - 1
        if i + 1 < len(items):
            nchunk, nsweep, nj, _ = items[i + 1]
            issued[i + 1] = {"x"} | ({"h"} if nsweep and not late else set())
            assert (i + 1) % 2 != i % 2
            if nsweep and not late:
                assert (nchunk, nj) in done_fwd, f"rows of tile {nj} copied before written"
        if not sweep:
            done_fwd.add((chunk, j))
        if late and i + 1 < len(items):
            issued[i + 1].add("h")  # after the barrier: every forward tile of the chunk is done
            assert all((chunk, t) in done_fwd for t in range(nt))


@pytest.mark.parametrize("nts", CKPT_CHUNKS)
def test_complex_checkpointed_copy_schedule(nts):
    ckpt_copy_schedule(nts)


def test_an_early_trajectory_copy_is_caught():
    with pytest.raises(AssertionError):
        ckpt_copy_schedule([3], defer=False)  # the first sweep item's rows before they exist
