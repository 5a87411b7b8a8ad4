"""Pins for the oracle's Flash PD-SSM scan (hard selection, one-hot column dictionary matrices
times a diagonal, straight-through backward).

Independent routes to the same numbers:
* finite-state-automaton emulation ("Flash PD-SSM", Proposition 1 as summarised: a single layer of
  size N represents any deterministic N-state automaton exactly): with d = 1, bt = 0 and h0 the
  start state's one-hot vector, the state is the one-hot vector of the automaton's state after
  every step, for modular counting and for a random transition table;
* dense brute force: A_t = P_{k_t} D_t built as an N x N matrix, h_t = A_t h_{t-1} + bt_t;
* PyTorch autograd through the dense form with the straight-through construction
  A_t = (P_hard + P_soft - stop_gradient(P_soft)) D_t, P_soft = sum_k softmax(scores/tau)_k P_k,
  which is the hard matrix in value and the tempered softmax in gradient;
* central finite differences in d, bt and h0 (the selection does not move);
* ties in the scores pick the lowest index.
"""

import numpy as np
import pytest
import torch

from selective_state_space_bwd_b200 import inputs as gen


def _dense_P(dictionary, k, N):
    P = np.zeros((N, N))
    P[dictionary[k], np.arange(N)] = 1.0
    return P


def _automaton_inputs(table, symbols, N, K):
    """table[k, j]: next state from state j on symbol k."""
    B, L = symbols.shape
    scores = np.full((B, L, 1, K), -1.0)
    scores[np.arange(B)[:, None], np.arange(L)[None, :], 0, symbols] = 10.0
    d = np.ones((B, L, 1, N))
    bt = np.zeros((B, L, 1, N))
    h0 = np.zeros((B, 1, N))
    h0[:, 0, 0] = 1.0
    return scores, d, bt, h0


@pytest.mark.parametrize("kind", ["modular", "random"])
def test_automaton_emulation(oracle_mod, kind):
    N, K, B, L = 8, 5, 3, 200
    rng = np.random.default_rng(4)
    if kind == "modular":
        table = (np.arange(N)[None, :] + np.arange(K)[:, None]) % N
    else:
        table = rng.integers(0, N, size=(K, N))
    symbols = rng.integers(0, K, size=(B, L))
    scores, d, bt, h0 = _automaton_inputs(table, symbols, N, K)
    o = oracle_mod.pdssm(scores, table.astype(np.int32), d, bt, h0, threads=1)
    for b in range(B):
        q = 0
        for t in range(L):
            q = table[symbols[b, t], q]
            expect = np.zeros(N)
            expect[q] = 1.0
            np.testing.assert_array_equal(o["h"][b, t, 0], expect)
    np.testing.assert_array_equal(o["sel"][:, :, 0], symbols)


def test_dense_brute_force_and_selection(oracle_mod):
    c = gen.pdssm_inputs(2, 30, 3, 8, 5, seed=2)
    o = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"], c["h0"], threads=1)
    B, L, H, K = c["scores"].shape
    N = c["d"].shape[-1]
    for b in range(B):
        for e in range(H):
            h = c["h0"][b, e].astype(np.float64)
            for t in range(L):
                k = int(np.argmax(c["scores"][b, t, e]))
                assert o["sel"][b, t, e] == k
                A = _dense_P(c["dictionary"], k, N) @ np.diag(c["d"][b, t, e].astype(np.float64))
                h = A @ h + c["bt"][b, t, e]
                np.testing.assert_allclose(o["h"][b, t, e], h, rtol=1e-13, atol=1e-13)


def test_ties_pick_the_lowest_index(oracle_mod):
    c = gen.pdssm_inputs(1, 4, 1, 4, 3, seed=3)
    c["scores"][:] = 0.0
    c["scores"][0, 1, 0] = [2.0, 2.0, 1.0]
    c["scores"][0, 2, 0] = [1.0, 3.0, 3.0]
    o = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"], c["h0"], threads=1)
    assert list(o["sel"][0, :, 0]) == [0, 0, 1, 0]


@pytest.mark.parametrize("tau", [1.0, 0.25])
def test_straight_through_backward_matches_autograd(oracle_mod, tau):
    c = gen.pdssm_inputs(2, 12, 2, 4, 3, seed=5)
    o = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"], c["h0"], c["g"], tau=tau,
                         threads=1)
    B, L, H, K = c["scores"].shape
    N = c["d"].shape[-1]
    Pk = torch.stack([torch.from_numpy(_dense_P(c["dictionary"], k, N)) for k in range(K)])
    sc = torch.tensor(c["scores"], dtype=torch.float64, requires_grad=True)
    d = torch.tensor(c["d"], dtype=torch.float64, requires_grad=True)
    bt = torch.tensor(c["bt"], dtype=torch.float64, requires_grad=True)
    h0 = torch.tensor(c["h0"], dtype=torch.float64, requires_grad=True)
    g = torch.tensor(c["g"], dtype=torch.float64)
    loss = 0.0
    for b in range(B):
        for e in range(H):
            h = h0[b, e]
            for t in range(L):
                p = torch.softmax(sc[b, t, e] / tau, dim=0)
                P_soft = (p[:, None, None] * Pk).sum(0)
                P_hard = Pk[int(torch.argmax(sc[b, t, e]))]
                A = (P_hard + P_soft - P_soft.detach()) @ torch.diag(d[b, t, e])
                h = A @ h + bt[b, t, e]
                loss = loss + (g[b, t, e] * h).sum()
    loss.backward()
    for name, t in (("dscores", sc), ("dd", d), ("dbt", bt), ("dh0", h0)):
        np.testing.assert_allclose(o[name], t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_finite_differences_smooth_inputs(oracle_mod):
    c = gen.pdssm_inputs(2, 7, 2, 4, 3, seed=6)
    c = {k: (v.astype(np.float64) if v.dtype != np.int32 else v) for k, v in c.items()}
    o = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"], c["h0"], c["g"], threads=1)

    def loss():
        h = oracle_mod.pdssm(c["scores"], c["dictionary"], c["d"], c["bt"], c["h0"], threads=1)["h"]
        return float(np.sum(c["g"] * h))

    for name, gname in (("d", "dd"), ("bt", "dbt"), ("h0", "dh0")):
        fd = np.zeros_like(c[name])
        for idx in np.ndindex(c[name].shape):
            v = c[name][idx]
            eps = 1e-6 * max(1.0, abs(v))
            c[name][idx] = v + eps
            lp = loss()
            c[name][idx] = v - eps
            lm = loss()
            c[name][idx] = v
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - o[gname]) / np.linalg.norm(o[gname])
        assert err < 1e-8, (name, err)
