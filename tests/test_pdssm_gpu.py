"""GPU parity of the Flash PD-SSM scan (ssm_pdssm_fwd / ssm_pdssm_bwd) against the float64 oracle.

Tolerances (relative L2 per tensor): trajectory h 1e-5; gradients dd, dbt, dscores, dh0 1e-4;
the selection (argmax of the same float32 scores) and automaton emulation exactly."""

import numpy as np
import pytest
import torch

from selective_state_space_bwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu

FWD_TOL, GRAD_TOL = 1e-5, 1e-4


@pytest.fixture(scope="module")
def S():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from selective_state_space_bwd_b200 import build, ssm_scan
    build.build()
    ssm_scan.lib()
    return ssm_scan


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / den if den > 0 else np.linalg.norm(a.ravel())


def dev(c):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in c.items()}


def run(S, c, tau, with_h0=True):
    d = dev(c)
    h0 = d["h0"] if with_h0 else None
    h, sel = S.ssm_pdssm_fwd(d["scores"], d["dictionary"], d["d"], d["bt"], h0=h0)
    out = S.ssm_pdssm_bwd(d["scores"], d["dictionary"], d["d"], h, sel, d["g"], tau=tau, h0=h0)
    torch.cuda.synchronize()
    res = {"h": h.cpu().numpy(), "sel": sel.cpu().numpy()}
    res.update({k: v.cpu().numpy() for k, v in out.items()})
    return res


CASES = [  # B, L, H, N, K
    (2, 100, 13, 16, 8),
    (1, 37, 40, 4, 3),
    (3, 65, 17, 8, 1),
    (2, 130, 5, 32, 32),
    (1, 16, 32, 16, 5),
    (1, 1000, 8, 16, 8),   # few CTAs: 13 time segments (summaries, carries, rescans)
    (1, 300, 3, 4, 5),     # 4 segments, partial last segment
    (2, 257, 20, 8, 6),    # 2 segments
    (2, 150, 9, 4, 9),     # K * heads-per-CTA > 256: argmax and score gradient as kernels of their own
    (1, 200, 16, 8, 17),   # the same with N = 8
    (3, 96, 64, 32, 32),   # largest state and dictionary
]


@pytest.mark.parametrize("B,L,H,N,K", CASES)
@pytest.mark.parametrize("with_h0", [True, False])
def test_pdssm_matches_oracle(S, oracle_mod, B, L, H, N, K, with_h0):
    c = gen.pdssm_inputs(B, L, H, N, K, seed=B * 100 + L + H + N + K)
    tau = 0.5
    got = run(S, c, tau, with_h0)
    ref = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"],
                           c["h0"] if with_h0 else None, c["g"], tau=tau)
    np.testing.assert_array_equal(got["sel"], ref["sel"])
    assert rel(got["h"], ref["h"]) <= FWD_TOL
    for k in ("dd", "dbt", "dscores", "dh0"):
        assert rel(got[k], ref[k]) <= GRAD_TOL, (k, rel(got[k], ref[k]))


@pytest.mark.parametrize("N,K,B,L,H", [(16, 5, 2, 90, 11), (32, 3, 1, 70, 6), (8, 4, 2, 300, 40)])
def test_pdssm_high_in_degree(S, oracle_mod, N, K, B, L, H):
    """Dictionaries whose rows collect more than seven columns (all columns into one row, half of
    them into another) take the plain in-list gather instead of the packed words."""
    c = gen.pdssm_inputs(B, L, H, N, K, seed=N + K)
    c["dictionary"][0, :] = 0
    c["dictionary"][1, : N // 2] = N - 1
    got = run(S, c, 0.7)
    ref = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"], c["h0"], c["g"], tau=0.7)
    np.testing.assert_array_equal(got["sel"], ref["sel"])
    assert rel(got["h"], ref["h"]) <= FWD_TOL
    for k in ("dd", "dbt", "dscores", "dh0"):
        assert rel(got[k], ref[k]) <= GRAD_TOL, (k, rel(got[k], ref[k]))


def test_pdssm_automaton_emulation_exact(S):
    N, K, B, L, H = 16, 6, 2, 300, 3
    rng = np.random.default_rng(8)
    table = rng.integers(0, N, size=(K, N)).astype(np.int32)
    symbols = rng.integers(0, K, size=(B, L, H))
    scores = np.full((B, L, H, K), -1.0, dtype=np.float32)
    np.put_along_axis(scores, symbols[..., None], 10.0, axis=-1)
    c = dict(scores=scores, dictionary=table, d=np.ones((B, L, H, N), np.float32),
             bt=np.zeros((B, L, H, N), np.float32), h0=np.zeros((B, H, N), np.float32))
    c["h0"][:, :, 0] = 1.0
    d = dev(c)
    h, sel = S.ssm_pdssm_fwd(d["scores"], d["dictionary"], d["d"], d["bt"], h0=d["h0"])
    torch.cuda.synchronize()
    h = h.cpu().numpy()
    q = np.zeros((B, H), dtype=np.int64)
    for t in range(L):
        q = table[symbols[:, t, :], q]
        expect = np.zeros((B, H, N), np.float32)
        np.put_along_axis(expect, q[..., None], 1.0, axis=-1)
        np.testing.assert_array_equal(h[:, t], expect)
    np.testing.assert_array_equal(sel.cpu().numpy(), symbols)


def test_pdssm_deterministic(S):
    c = gen.pdssm_inputs(2, 200, 24, 16, 8, seed=3)
    a, b = run(S, c, 1.0), run(S, c, 1.0)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_pdssm_invalid_dictionary_flags_status(S):
    c = gen.pdssm_inputs(1, 20, 8, 8, 4, seed=4)
    c["dictionary"][2, 5] = 8  # out of [0, N)
    d = dev(c)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    S.ssm_pdssm_fwd(d["scores"], d["dictionary"], d["d"], d["bt"], ws=ws)
    assert S.ssm_scan_status(ws) == 1
    c["dictionary"][2, 5] = 7
    d = dev(c)
    S.ssm_pdssm_fwd(d["scores"], d["dictionary"], d["d"], d["bt"], ws=ws)
    assert S.ssm_scan_status(ws) == 0


def test_pdssm_empty_sequence(S):
    c = gen.pdssm_inputs(2, 0, 4, 8, 3, seed=5)
    got = run(S, c, 1.0)
    assert got["h"].size == 0 and not got["dh0"].any()


def test_pdssm_full_size_sampled_heads(S, oracle_mod):
    """The bench workload (B=8, L=5120, H=256, N=16, K=8) in one call; heads are independent, so the
    oracle checks a sample of them on their own."""
    w = gen.WORKLOADS["pdssm_l5120"]
    c = gen.pdssm_inputs(w.batch, w.seqlen, w.heads, w.nstate, w.ndict, seed=0)
    got = run(S, c, 1.0)
    hs = np.array([0, 1, 100, 254, 255])
    sub = {k: (v[:, :, hs] if k in ("scores", "d", "bt", "g") else v) for k, v in c.items()}
    sub["h0"] = c["h0"][:, hs]
    ref = oracle_mod.pdssm(sub["scores"], sub["dictionary"], sub["d"], sub["bt"], sub["h0"],
                           sub["g"], tau=1.0)
    assert rel(got["h"][:, :, hs], ref["h"]) <= FWD_TOL
    for k in ("dd", "dbt", "dscores"):
        assert rel(got[k][:, :, hs], ref[k]) <= GRAD_TOL, k
    assert rel(got["dh0"][:, hs], ref["dh0"]) <= GRAD_TOL
