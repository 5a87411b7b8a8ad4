"""GPU parity of exact structured RTRL (ssm_scan_complex_rtrl) against the float64 oracle's
RTRL, and against the GPU's own reverse-time adjoint.  Tolerances (relative L2): trajectory h and
the carried state 1e-5, the gradients dlambda / domega 1e-4 (complex64 I/O)."""

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
    a, b = np.asarray(a, np.complex128), np.asarray(b, np.complex128)
    den = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / den if den > 0 else np.linalg.norm(a.ravel())


def dev(c):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in c.items()}


@pytest.mark.parametrize("B,L,K", [(2, 300, 128), (1, 1000, 64), (3, 17, 66), (2, 1, 64)])
def test_rtrl_matches_oracle(S, oracle_mod, B, L, K):
    c = gen.complex_inputs(B, L, K, seed=B + L + K)
    d = dev(c)
    st0 = (np.random.default_rng(5).standard_normal((B, 3, K, 2)) * 0.5).astype(np.float32)
    st0 = st0[..., 0] + 1j * st0[..., 1]
    state = torch.from_numpy(st0.astype(np.complex64)).cuda()
    got = S.ssm_scan_complex_rtrl(d["u"], d["r"], d["phi"], d["lam"], d["omega"], d["g"],
                                  state=state, want_h=True)
    torch.cuda.synchronize()
    ref = oracle_mod.complex_rtrl(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"],
                                  state=st0.astype(np.complex64), want_h=True)
    assert rel(got["h"].cpu().numpy(), ref["h"]) <= FWD_TOL
    assert rel(state.cpu().numpy(), ref["state"]) <= FWD_TOL
    for k in ("dlambda", "domega"):
        assert rel(got[k].cpu().numpy(), ref[k]) <= GRAD_TOL, k


def test_rtrl_matches_gpu_adjoint(S):
    c = gen.complex_inputs(2, 2048, 256, seed=9)
    d = dev(c)
    rt = S.ssm_scan_complex_rtrl(d["u"], d["r"], d["phi"], d["lam"], d["omega"], d["g"])
    h = S.ssm_scan_complex_fwd(d["u"], d["r"], d["phi"], d["lam"], d["omega"])
    adj = S.ssm_scan_complex_bwd_traj(h, d["r"], d["phi"], d["lam"], d["omega"], d["g"])
    torch.cuda.synchronize()
    for k in ("dlambda", "domega"):
        assert rel(rt[k].cpu().numpy(), adj[k].cpu().numpy()) <= GRAD_TOL, k


def test_rtrl_streaming_two_calls_equal_one(S):
    B, L, K, L1 = 2, 700, 128, 300
    c = gen.complex_inputs(B, L, K, seed=21)
    d = dev(c)
    one_state = torch.zeros((B, 3, K), dtype=torch.complex64, device="cuda")
    one = S.ssm_scan_complex_rtrl(d["u"], d["r"], d["phi"], d["lam"], d["omega"], d["g"],
                                  state=one_state)
    st = torch.zeros_like(one_state)
    parts = []
    for lo, hi in ((0, L1), (L1, L)):
        sl = {k: (v[:, lo:hi].contiguous() if v.dim() >= 2 else v) for k, v in d.items()}
        parts.append(S.ssm_scan_complex_rtrl(sl["u"], sl["r"], sl["phi"], d["lam"], d["omega"],
                                             sl["g"], state=st))
    torch.cuda.synchronize()
    for k in ("dlambda", "domega"):
        tot = parts[0][k].double() + parts[1][k].double()
        assert rel(tot.cpu().numpy(), one[k].cpu().numpy()) <= GRAD_TOL, k
    assert rel(st.cpu().numpy(), one_state.cpu().numpy()) <= FWD_TOL


def test_rtrl_full_size_sampled_modes(S, oracle_mod):
    """The complex workload (B=16, L=4096, K=2048) in one call; modes are independent, so the oracle
    checks a sample of them on their own columns."""
    w = gen.WORKLOADS["sparc_complex"]
    c = gen.complex_inputs(w.batch, w.seqlen, w.modes, seed=0)
    d = dev(c)
    got = S.ssm_scan_complex_rtrl(d["u"], d["r"], d["phi"], d["lam"], d["omega"], d["g"])
    torch.cuda.synchronize()
    ks = np.array([0, 1, 63, 64, 777, 1024, 2046, 2047])
    ref = oracle_mod.complex_rtrl(c["u"][:, :, ks], c["r"], c["phi"], c["lam"][ks],
                                  c["omega"][ks], c["g"][:, :, ks])
    for k in ("dlambda", "domega"):
        assert rel(got[k].cpu().numpy()[ks], ref[k]) <= GRAD_TOL, k


def test_rtrl_empty_sequence(S):
    c = gen.complex_inputs(2, 0, 64, seed=1)
    d = dev(c)
    state = torch.randn((2, 3, 64), dtype=torch.complex64, device="cuda")
    before = state.clone()
    got = S.ssm_scan_complex_rtrl(d["u"], d["r"], d["phi"], d["lam"], d["omega"], d["g"],
                                  state=state)
    torch.cuda.synchronize()
    assert not got["dlambda"].any() and not got["domega"].any()
    assert torch.equal(state, before)


def test_rtrl_far_phases(S, oracle_mod):
    """Phases beyond the pi/2 reduction's range go through the library sine/cosine."""
    c = gen.complex_inputs(2, 150, 64, seed=12)
    c["phi"][0, 10:20] = np.linspace(-8000.0, 8000.0, 10, dtype=np.float32)
    d = dev(c)
    got = S.ssm_scan_complex_rtrl(d["u"], d["r"], d["phi"], d["lam"], d["omega"], d["g"])
    torch.cuda.synchronize()
    ref = oracle_mod.complex_rtrl(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"])
    for k in ("dlambda", "domega"):
        assert rel(got[k].cpu().numpy(), ref[k]) <= GRAD_TOL, k
