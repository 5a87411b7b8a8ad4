"""Pins for the oracle's step-size projection (delta_raw = u w^T + bias) and its gradient.

Independent routes: numpy's matrix product (a library routine, not the oracle's loops); central
finite differences of a linear loss; the identity map (R = D, w = I: delta_raw = u + bias); and
the composition with the scan oracle, where the chain rule through the projection (ddelta_raw
from the scan's adjoint, then the projection's backward) must equal finite differences of the
scan's loss in u, w and bias.
"""

import numpy as np
import pytest

from selective_state_space_bwd_b200 import inputs as gen


@pytest.mark.parametrize("M,D,R", [(7, 24, 16), (1, 1, 1), (33, 8, 48), (5, 40, 3)])
def test_matches_numpy_matmul(oracle_mod, M, D, R):
    rng = np.random.default_rng(M + D + R)
    u, w, b, g = (rng.standard_normal(s) for s in ((M, R), (D, R), (D,), (M, D)))
    o = oracle_mod.dtproj(u, w, b, g)
    np.testing.assert_allclose(o["delta_raw"], u @ w.T + b, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o["du"], g @ w, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o["dw"], g.T @ u, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o["dbias"], g.sum(0), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(oracle_mod.dtproj(u, w)["delta_raw"], u @ w.T, rtol=1e-13, atol=1e-13)


def test_identity_map(oracle_mod):
    rng = np.random.default_rng(1)
    u = rng.standard_normal((3, 4, 6))
    b = rng.standard_normal(6)
    o = oracle_mod.dtproj(u, np.eye(6), b)
    np.testing.assert_array_equal(o["delta_raw"], u + b)


def test_finite_differences_linear_loss(oracle_mod):
    rng = np.random.default_rng(2)
    M, D, R = 4, 5, 3
    u, w, b, g = (rng.standard_normal(s) for s in ((M, R), (D, R), (D,), (M, D)))
    o = oracle_mod.dtproj(u, w, b, g)
    for name, arr, grad in (("u", u, o["du"]), ("w", w, o["dw"]), ("bias", b, o["dbias"])):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            v = arr[idx]
            arr[idx] = v + 1e-3
            lp = np.sum(g * oracle_mod.dtproj(u, w, b)["delta_raw"])
            arr[idx] = v - 1e-3
            lm = np.sum(g * oracle_mod.dtproj(u, w, b)["delta_raw"])
            arr[idx] = v
            fd[idx] = (lp - lm) / 2e-3
        np.testing.assert_allclose(fd, grad, rtol=1e-9, atol=1e-9, err_msg=name)


def test_composition_with_the_scan(oracle_mod):
    """loss = sum dy * y(scan(x, delta_raw = u w^T + bias, ...)): the projection's backward fed
    with the scan's ddelta_raw equals finite differences of the loss in u, w and bias."""
    B, L, D, N, R = 1, 12, 3, 4, 2
    c = gen.real_inputs(B, L, D, N, kind="mamba", seed=3)
    p = gen.dtproj_inputs(B, L, D, R, seed=4)
    u, w, b = (p[k].astype(np.float64) for k in ("u", "w", "bias"))

    def loss(u, w, b):
        dr = oracle_mod.dtproj(u, w, b)["delta_raw"]
        y = oracle_mod.real(c["x"], dr, c["A_log"], c["Bm"], c["Cm"], c["Dskip"], chunk=16)["y"]
        return float(np.sum(c["dy"] * y))

    dr = oracle_mod.dtproj(u, w, b)["delta_raw"]
    sc = oracle_mod.real(c["x"], dr, c["A_log"], c["Bm"], c["Cm"], c["Dskip"], c["dy"], chunk=16)
    grads = oracle_mod.dtproj(u, w, b, sc["ddelta_raw"])
    for name, arr, grad in (("u", u, grads["du"]), ("w", w, grads["dw"]), ("bias", b, grads["dbias"])):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            v = arr[idx]
            eps = 1e-6
            arr[idx] = v + eps
            lp = loss(u, w, b)
            arr[idx] = v - eps
            lm = loss(u, w, b)
            arr[idx] = v
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - grad) / np.linalg.norm(grad)
        assert err < 1e-6, (name, err)
