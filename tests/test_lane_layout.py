"""Host model checks of the index arithmetic of the real kernels: the lanes of the backward's
dB / dC channel sums, the partition of its fused sums, and the sub-tile walk of the segment
summaries.

A thread of the backward holds four states of one channel.  Its state slots are rotated by its
position `rot` among four neighbouring channel lanes (slot j holds state n0 + ((j + rot) & 3)),
and after each step the four lanes run an all-to-all in three shuffle rounds, round k sending
slot k to the partner whose rotation is rot - k.  This test replays those index formulas (as
written in csrc/real_bwd.cu) for every lane of a warp and every supported state size and checks
that each lane ends with the sum over its group's four channels of one state, that the four lanes
of a group cover the group's four states, and that the shared-memory layout of the window sums
is free of bank conflicts on both the writes and the reads.
"""

import itertools
import numpy as np
import pytest


def lane_layout(N):
    NG = N // 4
    out = []
    for lane in range(32):
        ng, cl = lane % NG, lane // NG
        rot = cl & 3
        n0 = 4 * ng
        srcs = [ng + NG * ((cl & ~3) | ((rot - k) & 3)) for k in (1, 2, 3)]
        sidx = [n0 + ((j + rot) & 3) for j in range(4)]
        out.append(dict(ng=ng, cl=cl, rot=rot, n0=n0, srcs=srcs, sidx=sidx))
    return NG, out


@pytest.mark.parametrize("N", [4, 8, 16])
def test_all_to_all_sums_each_state_over_its_group(N):
    NG, lay = lane_layout(N)
    rng = np.random.default_rng(N)
    val = rng.normal(size=(32 // NG, N))  # value[channel lane][state]
    slot = np.array([[val[L["cl"], s] for s in L["sidx"]] for L in lay])
    for lane, L in enumerate(lay):
        got = slot[lane, 0] + sum(slot[src, k + 1] for k, src in enumerate(L["srcs"]))
        # every source lane is in the same state group and the same four-channel group
        for src in L["srcs"]:
            assert lay[src]["ng"] == L["ng"] and lay[src]["cl"] // 4 == L["cl"] // 4
        group = [(L["cl"] & ~3) + i for i in range(4)]
        want = sum(val[c, L["n0"] + L["rot"]] for c in group)
        assert got == pytest.approx(want, rel=1e-12, abs=1e-12)
    # the four lanes of a group hold the group's four states, one each
    for ng in range(NG):
        for c0 in range(0, 32 // NG, 4):
            states = sorted(L["n0"] + L["rot"] for L in lay if L["ng"] == ng and L["cl"] // 4 == c0 // 4)
            assert states == list(range(4 * ng, 4 * ng + 4))


def banks(addrs):
    """Shared-memory wavefronts of one warp-wide 4-byte access (distinct words per bank)."""
    per_bank = {}
    for a in set(addrs):
        per_bank.setdefault(a % 32, set()).add(a)
    return max(len(v) for v in per_bank.values())


@pytest.mark.parametrize("N", [4, 8, 16])
def test_window_sums_layout_is_conflict_free(N):
    NG, lay = lane_layout(N)
    W, DT = 4, 32
    NT = DT * NG
    RS, GRP, N2 = 9 * N, DT // 4, 2 * N
    assert W * N2 == NT
    for warp in range(NT // 32):
        for u in range(W):
            for kind in range(2):
                addrs = []
                for lane, L in enumerate(lay):
                    dl = (warp * 32 + lane) // NG
                    grp = dl >> 2
                    addrs.append(grp * RS + u * N2 + kind * N + L["n0"] + L["rot"])
                assert banks(addrs) == 1
        # the readers: thread tid sums red[g * RS + tid] over the groups
        for g in range(GRP):
            assert banks([g * RS + warp * 32 + lane for lane in range(32)]) == 1


@pytest.mark.parametrize("N", [4, 8, 16])
def test_fused_dbc_share_partition(N):
    """Model of the backward's fused dB/dC sums (fused_dbc_share in real_bwd.cu): channel tile dt
    of a batch row sums rows [rows*dt/ndt, rows*(dt+1)/ndt) of a chunk; the share's float4 units
    times P = threads / units parts of the tiles spread over the CTA's threads.  Every output of
    the chunk is written exactly once, and every tile's partial of it is read exactly once."""
    N2, U4 = 2 * N, 2 * N // 4
    NT = 32 * N // 4
    for ndt, rows in itertools.product((1, 3, 32, 48, 128), (1, 5, 16, 127, 128)):
        written, reads = {}, {}
        for dt in range(ndt):
            r0, r1 = rows * dt // ndt, rows * (dt + 1) // ndt
            U = (r1 - r0) * U4
            for ub in range(0, U, NT):
                nu = min(NT, U - ub)
                P = NT // nu
                tp = (ndt + P - 1) // P
                for tid in range(NT):
                    unit, pq = tid % nu, tid // nu
                    u = ub + unit
                    if pq < P:
                        j0 = min(ndt, pq * tp)
                        for j in range(j0, min(ndt, j0 + tp)):
                            key = (j, r0 + u // U4, (u % U4) * 4)
                            reads[key] = reads.get(key, 0) + 1
                    if pq == 0:
                        for k in range(4):
                            o = (r0 + u // U4, (u % U4) * 4 + k)
                            written[o] = written.get(o, 0) + 1
        assert written == {(r, e): 1 for r in range(rows) for e in range(N2)}
        assert reads == {(j, r, e): 1 for j in range(ndt) for r in range(rows) for e in range(0, N2, 4)}


def summary_subtiles(L, T, seg_chunks, seg, TS, U):
    """The sub-tile walk of a segment summary, as the backward summary kernel
    (`real_bwd_summary_kernel`, TS = 32, U = 4) and the forward's summary instance (TS = min(T,
    32), U = 16) index it: (t0, rows, rows4) of sub-tiles k = 0..nsub-1 and, for the backward's
    three-stage ring, the raw stage each one occupies."""
    nC = -(-L // T)
    t_begin = seg * seg_chunks * T
    t_end = min(L, min(nC, (seg + 1) * seg_chunks) * T)
    nsub = -(-(t_end - t_begin) // TS) if t_end > t_begin else 0
    tiles = []
    for k in range(nsub):
        t0 = t_begin + k * TS
        rows = min(TS, t_end - t0)
        rows4 = -(-rows // U) * U
        tiles.append((t0, rows, rows4, k % 3))
    return t_begin, t_end, tiles


@pytest.mark.parametrize("T", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("TS,U", [(32, 4), ("fwd", 16)])
def test_segment_summary_subtiles_cover_each_step_once(T, TS, U):
    """Every step of a summarised segment lies in exactly one sub-tile; the rounding of a
    sub-tile to whole U-step groups stays inside the staged tile (32 rows) and reaches only past
    the sequence end, where the copies read zeros (so the rounded steps, with delta = 0, change
    nothing); and in the backward's ring the stage a sub-tile's copies are issued into (two
    ahead, k - 2, walking k downwards) is the one the sub-tile processed just before (k + 1)
    occupied."""
    ts = min(T, 32) if TS == "fwd" else TS
    for L, sc in itertools.product((1, 15, 16, 17, 100, 257, 1000, 4099), (1, 2, 3, 7)):
        nseg = -(-(-(-L // T)) // sc)
        for seg in range(1, nseg):
            t_begin, t_end, tiles = summary_subtiles(L, T, sc, seg, ts, U)
            covered = []
            for t0, rows, rows4, _ in tiles:
                assert 0 < rows <= ts and rows4 <= 32
                covered.extend(range(t0, t0 + rows))
                assert all(t >= L for t in range(t0 + rows, t0 + rows4))
            assert covered == list(range(t_begin, t_end))
            if TS != "fwd":
                for k in range(2, len(tiles) - 1):
                    assert tiles[k - 2][3] == tiles[k + 1][3]
