"""Pins for the float64 oracle: things fixed by the mathematics, not by the oracle itself.

Each pin is an independent route to the same number, chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand) fails at least one:

* hand-worked examples (tests/golden/worked_examples.json);
* the impulse response and the full unrolled (non-recurrent) sum h_t = sum_s (prod a) b_s;
* the geometric series for constant inputs and its steady state b / (1 - a);
* L = 1 by hand, forward and every gradient;
* central finite differences of the loss for every input entry (float64);
* PyTorch autograd through the unrolled sum (a different formulation, differentiated mechanically);
* Euler homogeneity identities (y is linear in x, in Bm, in Cm);
* the complex mode reducing to the real mode when omega = 0.
Softplus in these tests is numpy's ``logaddexp(0, z)``, an independent library routine.
"""

import json
import math
import os

import numpy as np
import pytest

from selective_state_space_bwd_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
LN2 = math.log(2.0)


def _poly_ln2(c):
    c = np.asarray(c, dtype=np.float64)
    return c[..., 0] + c[..., 1] * LN2 + c[..., 2] * LN2 * LN2


def _rand_real(B, L, D, N, seed, kind="mamba"):
    inp = gen.real_inputs(B, L, D, N, gen.F32, kind, seed)
    return {k: v.astype(np.float64) for k, v in inp.items()}


def _unrolled_h(inp):
    """h[b,t,d,n] = sum_{s<=t} exp(A_n (Lam_t - Lam_s)) delta_s Bm_s x_s, Lam = cumsum(delta)."""
    delta = np.logaddexp(0.0, inp["delta_raw"])  # [B,L,D]
    A = -np.exp(inp["A_log"])  # [D,N]
    lam = np.cumsum(delta, axis=1)  # [B,L,D]
    diff = lam[:, :, None, :] - lam[:, None, :, :]  # [B,t,s,D]
    L = delta.shape[1]
    mask = np.tril(np.ones((L, L)))[None, :, :, None]
    decay = np.exp(np.maximum(diff, 0.0)[..., None] * A[None, None, None]) * mask[..., None]
    bterm = (delta * inp["x"])[:, :, :, None] * inp["Bm"][:, :, None, :]  # [B,s,D,N]
    return np.einsum("btsdn,bsdn->btdn", decay, bterm)


def _y_from_h(inp, h):
    return np.einsum("btdn,btn->btd", h, inp["Cm"]) + inp["Dskip"] * inp["x"]


# ----------------------------------------------------------------------------- worked examples

def test_worked_example_real(oracle_mod):
    ex = json.load(open(GOLDEN))["real_L3"]
    I = ex["inputs"]
    x = np.array(I["x"]).reshape(1, 3, 1)
    dr = np.array(I["delta_raw"]).reshape(1, 3, 1)
    A_log = (np.array(I["A_log_is_ln2_times"]) * LN2).reshape(1, 2)
    Bm = np.array(I["Bm"]).reshape(1, 3, 2)
    Cm = np.array(I["Cm"]).reshape(1, 3, 2)
    Dskip = np.array(I["Dskip"])
    dy = np.array(I["dy"]).reshape(1, 3, 1)
    out = oracle_mod.real(x, dr, A_log, Bm, Cm, Dskip, dy, chunk=2, threads=1)
    E = ex["expected"]
    np.testing.assert_allclose(out["y"].ravel(), _poly_ln2(E["y"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["dx"].ravel(), _poly_ln2(E["dx"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["ddelta_raw"].ravel(), _poly_ln2(E["ddelta_raw"]),
                               rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["dB"].reshape(3, 2), _poly_ln2(E["dB"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["dC"].reshape(3, 2), _poly_ln2(E["dC"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["dA_log"].ravel(), _poly_ln2(E["dA_log"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["dD"], _poly_ln2(E["dD"]), rtol=1e-14, atol=1e-14)


def test_worked_example_complex(oracle_mod):
    ex = json.load(open(GOLDEN))["complex_L2"]
    I = ex["inputs"]
    u = np.array([complex(*p) for p in I["u"]]).reshape(1, 2, 1)
    g = np.array([complex(*p) for p in I["g"]]).reshape(1, 2, 1)
    r = np.array(I["r"]).reshape(1, 2)
    phi = np.array(I["phi"]).reshape(1, 2)
    lam = np.array(I["lambda"])
    om = np.array(I["omega_over_pi"]) * math.pi
    out = oracle_mod.complex_(u, r, phi, lam, om, g, threads=1)
    E = ex["expected"]
    np.testing.assert_allclose(out["h"].ravel(), [complex(*p) for p in E["h"]], atol=1e-15)
    np.testing.assert_allclose(out["du"].ravel(), [complex(*p) for p in E["du"]], atol=1e-15)
    np.testing.assert_allclose(out["dr"].ravel(), E["dr"], atol=1e-15)
    np.testing.assert_allclose(out["dphi"].ravel(), np.array(E["dphi_over_pi"]) * math.pi, atol=1e-15)
    np.testing.assert_allclose(out["dlambda"], np.array(E["dlambda_over_ln2"]) * LN2, atol=1e-15)
    np.testing.assert_allclose(out["domega"], E["domega"], atol=1e-15)


# ----------------------------------------------------------------------------- forward, real

@pytest.mark.parametrize("kind", ["mamba", "stiff"])
def test_impulse_response_closed_form(oracle_mod, kind):
    B, L, D, N = 2, 400, 3, 8
    inp = _rand_real(B, L, D, N, seed=1, kind=kind)
    inp["x"][:, 1:, :] = 0.0  # impulse at t = 0 only
    out = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                          inp["Dskip"], threads=2)
    delta = np.logaddexp(0.0, inp["delta_raw"])
    A = -np.exp(inp["A_log"])
    lam = np.cumsum(delta, axis=1) - delta[:, :1, :]  # sum_{s=1..t} delta_s
    h = np.exp(lam[..., None] * A[None, None]) * (delta[:, :1, :, None] * inp["Bm"][:, :1, None, :]
                                                 * inp["x"][:, :1, :, None])
    y = _y_from_h(inp, h)
    np.testing.assert_allclose(out["y"], y, rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("kind", ["mamba", "stiff"])
def test_unrolled_sum_and_checkpoints(oracle_mod, kind):
    B, L, D, N, T = 2, 70, 3, 4, 16
    inp = _rand_real(B, L, D, N, seed=2, kind=kind)
    out = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                          inp["Dskip"], chunk=T, threads=2, want_ckpt=True)
    h = _unrolled_h(inp)
    np.testing.assert_allclose(out["y"], _y_from_h(inp, h), rtol=1e-11, atol=1e-12)
    ends = [min((c + 1) * T, L) - 1 for c in range((L + T - 1) // T)]
    np.testing.assert_allclose(out["ckpt"], h[:, ends], rtol=1e-11, atol=1e-12)


def test_geometric_series_and_steady_state(oracle_mod):
    L, D, N = 3000, 2, 4
    x = np.full((1, L, D), 0.7)
    dr = np.full((1, L, D), -1.3)
    A_log = np.log(np.array([[0.5, 1.0, 2.0, 3.0], [0.1, 0.2, 0.3, 0.4]]))
    Bm = np.tile(np.array([1.0, -2.0, 0.5, 3.0]), (1, L, 1))
    Cm = np.zeros((1, L, N))
    Cm[..., 2] = 1.0  # y reads state n = 2 only
    Dskip = np.zeros(D)
    out = oracle_mod.real(x, dr, A_log, Bm, Cm, Dskip, threads=1)
    delta = np.logaddexp(0.0, -1.3)
    a = np.exp(-delta * np.exp(A_log[:, 2]))
    b = delta * 0.5 * 0.7
    t = np.arange(L)[:, None]
    expect = b * (1.0 - a ** (t + 1)) / (1.0 - a)
    np.testing.assert_allclose(out["y"][0], expect, rtol=1e-12)
    np.testing.assert_allclose(out["y"][0, -1], b / (1.0 - a), rtol=1e-10)


def test_L1_by_hand(oracle_mod):
    rng = np.random.default_rng(5)
    D, N = 3, 4
    x, dr, dy = (rng.standard_normal((1, 1, D)) for _ in range(3))
    A_log = rng.standard_normal((D, N))
    Bm, Cm = (rng.standard_normal((1, 1, N)) for _ in range(2))
    Dskip = rng.standard_normal(D)
    out = oracle_mod.real(x, dr, A_log, Bm, Cm, Dskip, dy, threads=1)
    delta = np.logaddexp(0.0, dr)[0, 0]
    cb = float(np.sum(Cm[0, 0] * Bm[0, 0]))
    xx, gy = x[0, 0], dy[0, 0]
    np.testing.assert_allclose(out["y"][0, 0], delta * cb * xx + Dskip * xx, rtol=1e-14)
    np.testing.assert_array_equal(out["dA_log"], np.zeros((D, N)))
    np.testing.assert_allclose(out["dx"][0, 0], Dskip * gy + delta * gy * cb, rtol=1e-14)
    sig = 1.0 / (1.0 + np.exp(-dr[0, 0]))
    np.testing.assert_allclose(out["ddelta_raw"][0, 0], gy * xx * cb * sig, rtol=1e-13)
    np.testing.assert_allclose(out["dB"][0, 0], Cm[0, 0] * np.sum(gy * delta * xx), rtol=1e-13)
    np.testing.assert_allclose(out["dC"][0, 0], Bm[0, 0] * np.sum(gy * delta * xx), rtol=1e-13)
    np.testing.assert_allclose(out["dD"], gy * xx, rtol=1e-14)


# ----------------------------------------------------------------------------- backward, real

def _real_loss(oracle_mod, inp, dy):
    o = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                        inp["Dskip"], threads=1)
    return float(np.sum(dy * o["y"]))


@pytest.mark.parametrize("kind", ["mamba", "stiff"])
def test_finite_differences_real(oracle_mod, kind):
    B, L, D, N = 2, 5, 3, 4
    inp = _rand_real(B, L, D, N, seed=3, kind=kind)
    dy = inp.pop("dy")
    out = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                          inp["Dskip"], dy, threads=1)
    names = {"x": "dx", "delta_raw": "ddelta_raw", "A_log": "dA_log", "Bm": "dB", "Cm": "dC",
             "Dskip": "dD"}
    for name, gname in names.items():
        fd = np.zeros_like(inp[name])
        for idx in np.ndindex(inp[name].shape):
            v = inp[name][idx]
            eps = 1e-6 * max(1.0, abs(v))
            inp[name][idx] = v + eps
            lp = _real_loss(oracle_mod, inp, dy)
            inp[name][idx] = v - eps
            lm = _real_loss(oracle_mod, inp, dy)
            inp[name][idx] = v
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - out[gname]) / max(np.linalg.norm(out[gname]), 1e-30)
        assert err < 1e-7, (name, err)


def test_autograd_through_unrolled_sum(oracle_mod):
    torch = pytest.importorskip("torch")
    B, L, D, N = 2, 24, 3, 4
    inp = _rand_real(B, L, D, N, seed=4, kind="mamba")
    dy = inp.pop("dy")
    out = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                          inp["Dskip"], dy, threads=1)
    T = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in inp.items()}
    delta = torch.nn.functional.softplus(T["delta_raw"])
    A = -torch.exp(T["A_log"])
    lam = torch.cumsum(delta, 1)
    diff = (lam[:, :, None, :] - lam[:, None, :, :]).clamp(min=0.0)
    mask = torch.tril(torch.ones(L, L, dtype=torch.float64))[None, :, :, None, None]
    decay = torch.exp(diff[..., None] * A) * mask
    bterm = (delta * T["x"])[..., None] * T["Bm"][:, :, None, :]
    h = torch.einsum("btsdn,bsdn->btdn", decay, bterm)
    y = torch.einsum("btdn,btn->btd", h, T["Cm"]) + T["Dskip"] * T["x"]
    (y * torch.tensor(dy)).sum().backward()
    pairs = {"x": "dx", "delta_raw": "ddelta_raw", "A_log": "dA_log", "Bm": "dB", "Cm": "dC",
             "Dskip": "dD"}
    for k, gk in pairs.items():
        np.testing.assert_allclose(out[gk], T[k].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=k)


def test_homogeneity_identities_real(oracle_mod):
    B, L, D, N = 2, 300, 8, 16
    inp = _rand_real(B, L, D, N, seed=6)
    o = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                        inp["Dskip"], inp["dy"], threads=2)
    loss = np.sum(inp["dy"] * o["y"])
    skip = np.sum(inp["dy"] * inp["Dskip"] * inp["x"])
    np.testing.assert_allclose(np.sum(inp["x"] * o["dx"]), loss, rtol=1e-11)
    np.testing.assert_allclose(np.sum(inp["Bm"] * o["dB"]), loss - skip, rtol=1e-11)
    np.testing.assert_allclose(np.sum(inp["Cm"] * o["dC"]), loss - skip, rtol=1e-11)
    np.testing.assert_allclose(np.sum(inp["Dskip"] * o["dD"]), skip, rtol=1e-12)


def test_channel_ranges_compose(oracle_mod):
    B, L, D, N = 2, 50, 6, 4
    inp = _rand_real(B, L, D, N, seed=7)
    args = (inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["dy"])
    full = oracle_mod.real(*args, threads=3)
    lo = oracle_mod.real(*args, d_range=(0, 2), threads=1)
    hi = oracle_mod.real(*args, d_range=(2, 6), threads=2)
    np.testing.assert_allclose(lo["dB"] + hi["dB"], full["dB"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lo["dC"] + hi["dC"], full["dC"], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(hi["y"][..., 2:], full["y"][..., 2:])
    assert np.isnan(hi["y"][..., :2]).all()


def test_empty_sequence(oracle_mod):
    D, N = 3, 4
    z = np.zeros((2, 0, D))
    o = oracle_mod.real(z, z, np.zeros((D, N)), np.zeros((2, 0, N)), np.zeros((2, 0, N)),
                        np.ones(D), z, threads=1)
    assert o["y"].shape == (2, 0, D)
    np.testing.assert_array_equal(o["dA_log"], 0.0)
    np.testing.assert_array_equal(o["dD"], 0.0)


# ----------------------------------------------------------------------------- complex mode

def _rand_complex(B, L, K, seed):
    c = gen.complex_inputs(B, L, K, seed)
    return {k: (v.astype(np.complex128) if np.iscomplexobj(v) else v.astype(np.float64))
            for k, v in c.items()}


def test_complex_impulse_and_unrolled_sum(oracle_mod):
    B, L, K = 2, 60, 5
    c = _rand_complex(B, L, K, seed=8)
    out = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], threads=2)
    s = np.logaddexp(0.0, c["r"])
    S, P = np.cumsum(s, 1), np.cumsum(c["phi"], 1)
    z = (-(S[:, :, None] - S[:, None, :])[..., None] * c["lam"]
         + 1j * (P[:, :, None] - P[:, None, :])[..., None] * c["omega"])  # [B,t,s,K]
    mask = np.tril(np.ones((L, L)))[None, :, :, None]
    h = np.einsum("btsk,bsk->btk", np.exp(z) * mask, c["u"])
    np.testing.assert_allclose(out["h"], h, rtol=1e-11, atol=1e-12)
    # impulse: only u_0 nonzero
    u0 = np.zeros_like(c["u"])
    u0[:, 0] = c["u"][:, 0]
    o2 = oracle_mod.complex_(u0, c["r"], c["phi"], c["lam"], c["omega"], threads=1)
    e = np.exp(-(S - s[:, :1])[..., None] * c["lam"] + 1j * (P - c["phi"][:, :1])[..., None] * c["omega"])
    np.testing.assert_allclose(o2["h"], e * u0[:, :1], rtol=1e-12, atol=1e-14)


def _complex_loss(oracle_mod, c):
    o = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], threads=1)
    return float(np.real(np.sum(np.conj(c["g"]) * o["h"])))


def test_finite_differences_complex(oracle_mod):
    B, L, K = 2, 6, 3
    c = _rand_complex(B, L, K, seed=9)
    out = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"], threads=1)
    for name, gname in [("r", "dr"), ("phi", "dphi"), ("lam", "dlambda"), ("omega", "domega")]:
        fd = np.zeros_like(c[name])
        for idx in np.ndindex(c[name].shape):
            v = c[name][idx]
            eps = 1e-6 * max(1.0, abs(v))
            c[name][idx] = v + eps
            lp = _complex_loss(oracle_mod, c)
            c[name][idx] = v - eps
            lm = _complex_loss(oracle_mod, c)
            c[name][idx] = v
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - out[gname]) / np.linalg.norm(out[gname])
        assert err < 1e-7, (name, err)
    fd = np.zeros_like(c["u"])
    for idx in np.ndindex(c["u"].shape):
        v = c["u"][idx]
        for part, unit in ((0, 1.0), (1, 1j)):
            eps = 1e-6
            c["u"][idx] = v + eps * unit
            lp = _complex_loss(oracle_mod, c)
            c["u"][idx] = v - eps * unit
            lm = _complex_loss(oracle_mod, c)
            c["u"][idx] = v
            fd[idx] += unit * (lp - lm) / (2 * eps)
    err = np.linalg.norm(fd - out["du"]) / np.linalg.norm(out["du"])
    assert err < 1e-7, err


def test_complex_homogeneity(oracle_mod):
    c = _rand_complex(2, 200, 16, seed=10)
    o = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"], threads=2)
    loss = np.real(np.sum(np.conj(c["g"]) * o["h"]))
    np.testing.assert_allclose(np.real(np.sum(np.conj(o["du"]) * c["u"])), loss, rtol=1e-11)


def test_complex_reduces_to_real_when_omega_zero(oracle_mod):
    """omega = 0 and real u: a = exp(-lambda softplus(r)) is the real mode with N = 1,
    A_log = log(lambda), delta_raw = r, Bm = 1/softplus(r), Cm = 1, Dskip = 0, x = u, dy = g."""
    B, L, K = 2, 80, 3
    c = _rand_complex(B, L, K, seed=11)
    u = c["u"].real.astype(np.complex128)
    g = c["g"].real.astype(np.complex128)
    om = np.zeros(K)
    co = oracle_mod.complex_(u, c["r"], c["phi"], c["lam"], om, g, threads=1)
    s = np.logaddexp(0.0, c["r"])
    for k in range(K):
        x = u[..., k].real[..., None]
        dr = c["r"][..., None]
        Bm = (1.0 / s)[..., None]
        Cm = np.ones((B, L, 1))
        ro = oracle_mod.real(x, dr, np.log(c["lam"][k:k + 1])[:, None], Bm, Cm, np.zeros(1),
                             g[..., k].real[..., None], threads=1)
        np.testing.assert_allclose(co["h"][..., k].real, ro["y"][..., 0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(co["h"][..., k].imag, 0.0, atol=1e-300)
        np.testing.assert_allclose(co["du"][..., k].real, ro["dx"][..., 0], rtol=1e-12, atol=1e-14)
        # dlambda = dL/dlambda = -dL/dA, and dA_log = A dL/dA with A = -lambda
        np.testing.assert_allclose(co["dlambda"][k], ro["dA_log"][0, 0] / c["lam"][k], rtol=1e-11)
    # dr (retention path only) = ddelta_raw minus its input-path part sigmoid(r) x Bm g,
    # summed over the modes; here each mode is a separate real problem
    total = np.zeros((B, L))
    for k in range(K):
        x = u[..., k].real
        ro = oracle_mod.real(x[..., None], c["r"][..., None], np.log(c["lam"][k:k + 1])[:, None],
                             (1.0 / s)[..., None], np.ones((B, L, 1)), np.zeros(1),
                             g[..., k].real[..., None], threads=1)
        sig = 1.0 / (1.0 + np.exp(-c["r"]))
        total += ro["ddelta_raw"][..., 0] - sig * x * (1.0 / s) * ro["dx"][..., 0]
    np.testing.assert_allclose(co["dr"], total, rtol=1e-10, atol=1e-12)
