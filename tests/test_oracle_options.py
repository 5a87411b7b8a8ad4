"""Pins for the oracle's real-mode options: initial state h0 / final state hL (with the gradients
dh0 and the upstream dhL), and the zero-order-hold input term of the blog's §1.1
(B̄ = (delta A)^-1 (exp(delta A) - 1) delta B, i.e. phi = expm1(delta A) / A per state).

Independent routes to the same numbers:

* the free response h_t = exp(A Lam_t) h0 (Lam = cumsum(delta)), no recurrence;
* for zero-order hold with B and x held constant, the exact solution of dh/dt = A h + B x over
  the time Lam_t: h_t = h* + exp(A Lam_t) (h0 - h*), h* = -B x / A;
* the unrolled (non-recurrent) sum with the zero-order-hold input term;
* the closed form of dh0 as a sum of decayed C dy terms plus the decayed dhL;
* L = 1 by hand for every gradient under zero-order hold;
* central finite differences of L = sum dy y + sum dhL hL for every input, h0 included;
* homogeneity: (y, hL) is linear in (x, h0) jointly.
numpy's ``logaddexp(0, z)`` and ``expm1`` are the independent library routines.
"""

import numpy as np
import pytest

from selective_state_space_bwd_b200 import inputs as gen


def _inputs(B, L, D, N, seed, kind="mamba"):
    inp = {k: v.astype(np.float64) for k, v in gen.real_inputs(B, L, D, N, gen.F32, kind, seed).items()}
    rng = np.random.default_rng(seed + 1000)
    inp["h0"] = rng.standard_normal((B, D, N))
    inp["dhL"] = rng.standard_normal((B, D, N))
    return inp


def _run(o, inp, zoh, with_dy=True, chunk=4, **kw):
    return o.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"], inp["Dskip"],
                  inp["dy"] if with_dy else None, chunk=chunk, threads=1, zoh=zoh,
                  h0=inp.get("h0"), dhL=inp.get("dhL") if with_dy else None, **kw)


def _lam(inp):
    return np.cumsum(np.logaddexp(0.0, inp["delta_raw"]), axis=1)  # [B,L,D]


@pytest.mark.parametrize("zoh", [False, True])
def test_free_response_closed_form(oracle_mod, zoh):
    inp = _inputs(2, 11, 3, 4, seed=5)
    inp["x"][:] = 0.0
    o = _run(oracle_mod, inp, zoh, with_dy=False)
    A = -np.exp(inp["A_log"])
    h = np.exp(_lam(inp)[..., None] * A[None, None]) * inp["h0"][:, None]  # [B,L,D,N]
    y = np.einsum("btdn,btn->btd", h, inp["Cm"])
    np.testing.assert_allclose(o["y"], y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o["hL"], h[:, -1], rtol=1e-12, atol=1e-13)


def test_zoh_is_the_exact_solution_for_held_inputs(oracle_mod):
    B, L, D, N = 2, 40, 3, 4
    inp = _inputs(B, L, D, N, seed=7, kind="stiff")
    inp["Bm"][:] = inp["Bm"][:, :1]          # B_t held constant over time
    inp["x"][:] = inp["x"][:, :1]            # x_t held constant over time
    o = _run(oracle_mod, inp, True, with_dy=False)
    A = -np.exp(inp["A_log"])                                     # [D,N]
    hstar = -inp["Bm"][:, 0, None, :] * inp["x"][:, 0, :, None] / A[None]  # [B,D,N]
    h = hstar[:, None] + np.exp(_lam(inp)[..., None] * A) * (inp["h0"] - hstar)[:, None]
    y = np.einsum("btdn,btn->btd", h, inp["Cm"]) + inp["Dskip"] * inp["x"]
    np.testing.assert_allclose(o["y"], y, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(o["hL"], h[:, -1], rtol=1e-10, atol=1e-11)


def test_zoh_unrolled_sum(oracle_mod):
    inp = _inputs(2, 9, 3, 4, seed=9)
    o = _run(oracle_mod, inp, True, with_dy=False)
    delta = np.logaddexp(0.0, inp["delta_raw"])
    A = -np.exp(inp["A_log"])
    lam = np.cumsum(delta, axis=1)
    L = delta.shape[1]
    phi = np.expm1(delta[..., None] * A) / A                          # [B,L,D,N]
    bterm = phi * inp["Bm"][:, :, None, :] * inp["x"][..., None]
    diff = lam[:, :, None, :] - lam[:, None, :, :]                    # [B,t,s,D]
    mask = np.tril(np.ones((L, L)))[None, :, :, None, None]
    decay = np.exp(np.maximum(diff, 0.0)[..., None] * A) * mask
    h = np.einsum("btsdn,bsdn->btdn", decay, bterm)
    h = h + np.exp(lam[..., None] * A) * inp["h0"][:, None]
    y = np.einsum("btdn,btn->btd", h, inp["Cm"]) + inp["Dskip"] * inp["x"]
    np.testing.assert_allclose(o["y"], y, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("zoh", [False, True])
def test_dh0_closed_form(oracle_mod, zoh):
    inp = _inputs(2, 10, 3, 4, seed=11)
    o = _run(oracle_mod, inp, zoh)
    A = -np.exp(inp["A_log"])
    lam = _lam(inp)
    decay = np.exp(lam[..., None] * A)                                 # prod_{s<=t} a_s
    dh0 = np.einsum("btdn,btn,btd->bdn", decay, inp["Cm"], inp["dy"]) + decay[:, -1] * inp["dhL"]
    np.testing.assert_allclose(o["dh0"], dh0, rtol=1e-12, atol=1e-13)


def test_zoh_L1_by_hand(oracle_mod):
    inp = _inputs(2, 1, 3, 4, seed=13)
    o = _run(oracle_mod, inp, True)
    z = inp["delta_raw"][:, 0]                                         # [B,D]
    delta = np.logaddexp(0.0, z)
    sig = 1.0 / (1.0 + np.exp(-z))
    A = -np.exp(inp["A_log"])                                          # [D,N]
    a = np.exp(delta[..., None] * A)                                   # [B,D,N]
    phi = np.expm1(delta[..., None] * A) / A
    Bt, Ct = inp["Bm"][:, 0][:, None, :], inp["Cm"][:, 0][:, None, :]  # [B,1,N]
    x, dy, h0, dhL = inp["x"][:, 0], inp["dy"][:, 0], inp["h0"], inp["dhL"]
    h = a * h0 + phi * Bt * x[..., None]
    np.testing.assert_allclose(o["y"][:, 0], (Ct * h).sum(-1) + inp["Dskip"] * x, rtol=1e-13)
    np.testing.assert_allclose(o["hL"], h, rtol=1e-13)
    g = Ct * dy[..., None] + dhL                                       # dL/dh_0
    np.testing.assert_allclose(o["dx"][:, 0], inp["Dskip"] * dy + (g * phi * Bt).sum(-1), rtol=1e-12)
    ddelta = (g * (A * a * h0 + a * Bt * x[..., None])).sum(-1)
    np.testing.assert_allclose(o["ddelta_raw"][:, 0], ddelta * sig, rtol=1e-12)
    np.testing.assert_allclose(o["dB"][:, 0], (g * phi * x[..., None]).sum(1), rtol=1e-12)
    np.testing.assert_allclose(o["dC"][:, 0], (dy[..., None] * h).sum(1), rtol=1e-12)
    dA = (g * (delta[..., None] * a * h0 + Bt * x[..., None] * (delta[..., None] * a - phi) / A)).sum(0)
    np.testing.assert_allclose(o["dA_log"], A * dA, rtol=1e-12)
    np.testing.assert_allclose(o["dD"], (dy * x).sum(0), rtol=1e-12)
    np.testing.assert_allclose(o["dh0"], a * g, rtol=1e-13)


def _loss(oracle_mod, inp, zoh):
    o = _run(oracle_mod, inp, zoh, with_dy=False)
    return float(np.sum(inp["dy"] * o["y"]) + np.sum(inp["dhL"] * o["hL"]))


@pytest.mark.parametrize("zoh,kind", [(False, "mamba"), (True, "mamba"), (True, "stiff")])
def test_finite_differences_with_options(oracle_mod, zoh, kind):
    inp = _inputs(2, 5, 3, 4, seed=17, kind=kind)
    out = _run(oracle_mod, inp, zoh)
    names = {"x": "dx", "delta_raw": "ddelta_raw", "A_log": "dA_log", "Bm": "dB", "Cm": "dC",
             "Dskip": "dD", "h0": "dh0"}
    for name, gname in names.items():
        fd = np.zeros_like(inp[name])
        for idx in np.ndindex(inp[name].shape):
            v = inp[name][idx]
            eps = 1e-6 * max(1.0, abs(v))
            inp[name][idx] = v + eps
            lp = _loss(oracle_mod, inp, zoh)
            inp[name][idx] = v - eps
            lm = _loss(oracle_mod, inp, zoh)
            inp[name][idx] = v
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - out[gname]) / max(np.linalg.norm(out[gname]), 1e-30)
        assert err < 1e-7, (name, err)


@pytest.mark.parametrize("zoh", [False, True])
def test_homogeneity_in_x_and_h0(oracle_mod, zoh):
    inp = _inputs(2, 13, 3, 4, seed=19)
    o = _run(oracle_mod, inp, zoh)
    lhs = np.sum(inp["x"] * o["dx"]) + np.sum(inp["h0"] * o["dh0"])
    rhs = np.sum(inp["dy"] * o["y"]) + np.sum(inp["dhL"] * o["hL"])
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(rhs))


def test_defaults_match_the_plain_call_and_last_checkpoint(oracle_mod):
    inp = _inputs(2, 10, 3, 4, seed=23)
    plain = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                            inp["Dskip"], inp["dy"], chunk=4, threads=1, want_ckpt=True)
    for k in ("y", "dx", "ddelta_raw", "dA_log", "dB", "dC", "dD"):
        assert np.array_equal(plain[k], oracle_mod.real(
            inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"], inp["Dskip"],
            inp["dy"], chunk=4, threads=1, h0=np.zeros_like(inp["h0"]),
            dhL=np.zeros_like(inp["dhL"]))[k]), k
    np.testing.assert_array_equal(plain["hL"], plain["ckpt"][:, -1])


def test_empty_sequence_passes_the_state_through(oracle_mod):
    inp = _inputs(2, 0, 3, 4, seed=29)
    o = _run(oracle_mod, inp, True)
    np.testing.assert_array_equal(o["hL"], inp["h0"])
    np.testing.assert_array_equal(o["dh0"], inp["dhL"])
