"""Host-side checks of the Flash PD-SSM backward's shared-memory scratch layout (no GPU).

The score-gradient pass gives lane L of a warp the (step, head) entry divmod(L + 32 p, SPW), with
SPW = 32 / N heads per warp, and all lanes read mu at one dictionary offset i: state i of entry
(r, c) sits at r*RS + c*(N+1) + i with RS = SPW*(N+1).  The 32 addresses must fall in 32 distinct
banks (16 for N = 32, whose warp has 16 entries per tile), and the scan's stores (lane L of step r
to r*RS + L + L // N) must stay inside the tile's TT*RS floats.
"""

import pytest

TT = 16


@pytest.mark.parametrize("N", [4, 8, 16, 32])
def test_score_gradient_reads_are_bank_conflict_free(N):
    spw = 32 // N
    rs = spw * (N + 1)
    entries = TT * spw
    for p in range((entries + 31) // 32):
        lanes = [L for L in range(32) if L + 32 * p < entries]
        for i in range(N):
            banks = []
            for L in lanes:
                r, c = divmod(L + 32 * p, spw)
                banks.append((r * rs + c * (N + 1) + i) % 32)
            assert len(set(banks)) == len(lanes), (N, p, i)


@pytest.mark.parametrize("N", [4, 8, 16, 32])
def test_scan_stores_stay_in_the_tile(N):
    spw = 32 // N
    rs = spw * (N + 1)
    top = max(r * rs + L + L // N for r in range(TT) for L in range(32))
    assert top < TT * rs
    # and they are the (r, c, j) slots the score gradient reads
    for L in range(32):
        c, j = divmod(L, N)
        assert L + L // N == c * (N + 1) + j
