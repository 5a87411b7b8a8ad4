"""Pins for the oracle's exact structured RTRL (complex mode): forward-mode sensitivities of the
state to each mode's lambda and omega, and the online gradient of Re sum conj(g) h.

Independent routes to the same numbers:
* the reverse-time adjoint of the complex backward (a different method, pinned separately);
* central finite differences of the loss in lambda and omega;
* the impulse response, where h_t = exp(-lambda Sum s + i omega Sum phi) u_0 gives the
  sensitivities in closed form: dh_t/dlambda = -(s_1 + .. + s_t) h_t, dh_t/domega = i (phi_1 + ..
  + phi_t) h_t;
* streaming: two calls that hand the state (h and both sensitivities) over equal one call.
"""

import numpy as np
import pytest

from selective_state_space_bwd_b200 import inputs as gen


@pytest.mark.parametrize("B,L,K,seed", [(2, 50, 6, 1), (1, 300, 4, 2), (3, 1, 5, 3)])
def test_rtrl_equals_the_adjoint(oracle_mod, B, L, K, seed):
    c = gen.complex_inputs(B, L, K, seed=seed)
    adj = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"], threads=1)
    rt = oracle_mod.complex_rtrl(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"],
                                 want_h=True, threads=1)
    np.testing.assert_array_equal(rt["h"], adj["h"])
    for k in ("dlambda", "domega"):
        scale = np.abs(adj[k]).max()
        np.testing.assert_allclose(rt[k], adj[k], rtol=1e-11, atol=1e-12 * scale)
    np.testing.assert_array_equal(rt["state"][:, 0], adj["h"][:, -1])


def test_rtrl_finite_differences(oracle_mod):
    c = gen.complex_inputs(2, 12, 3, seed=7)
    c = {k: (v.astype(np.complex128) if np.iscomplexobj(v) else v.astype(np.float64)) for k, v in c.items()}
    rt = oracle_mod.complex_rtrl(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"], threads=1)

    def loss():
        h = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], threads=1)["h"]
        return float(np.real(np.sum(np.conj(c["g"]) * h)))

    for name, gname in (("lam", "dlambda"), ("omega", "domega")):
        fd = np.zeros_like(c[name])
        for i in range(c[name].size):
            v = c[name][i]
            eps = 1e-6 * max(1.0, abs(v))
            c[name][i] = v + eps
            lp = loss()
            c[name][i] = v - eps
            lm = loss()
            c[name][i] = v
            fd[i] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - rt[gname]) / np.linalg.norm(rt[gname])
        assert err < 1e-7, (name, err)


def test_rtrl_impulse_sensitivities_closed_form(oracle_mod):
    B, L, K = 2, 40, 5
    c = gen.complex_inputs(B, L, K, seed=11)
    u = np.zeros_like(c["u"])
    u[:, 0] = c["u"][:, 0]
    rt = oracle_mod.complex_rtrl(u, c["r"], c["phi"], c["lam"], c["omega"], c["g"], threads=1)
    s = np.logaddexp(0.0, c["r"].astype(np.float64))          # [B,L]
    ph = c["phi"].astype(np.float64)
    S, P = s[:, 1:].sum(1), ph[:, 1:].sum(1)                  # steps 1..L-1 act on u_0
    lam, om = c["lam"].astype(np.float64), c["omega"].astype(np.float64)
    h = np.exp(-lam * S[:, None] + 1j * om * P[:, None]) * u[:, 0].astype(np.complex128)
    st = rt["state"]
    np.testing.assert_allclose(st[:, 0], h, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(st[:, 1], -S[:, None] * h, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(st[:, 2], 1j * P[:, None] * h, rtol=1e-12, atol=1e-14)


def test_rtrl_streaming_two_calls_equal_one(oracle_mod):
    B, L, K, L1 = 2, 64, 4, 27
    c = gen.complex_inputs(B, L, K, seed=13)
    one = oracle_mod.complex_rtrl(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"], threads=1)
    a = oracle_mod.complex_rtrl(c["u"][:, :L1], c["r"][:, :L1], c["phi"][:, :L1], c["lam"],
                                c["omega"], c["g"][:, :L1], threads=1)
    b = oracle_mod.complex_rtrl(c["u"][:, L1:], c["r"][:, L1:], c["phi"][:, L1:], c["lam"],
                                c["omega"], c["g"][:, L1:], state=a["state"], threads=1)
    for k in ("dlambda", "domega"):
        np.testing.assert_allclose(a[k] + b[k], one[k], rtol=1e-11, atol=1e-12 * np.abs(one[k]).max())
    np.testing.assert_allclose(b["state"], one["state"], rtol=1e-12, atol=1e-13)
