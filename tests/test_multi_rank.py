"""Multi-rank data parallelism on CPU (gloo, world size 2): each rank takes its batch shard, runs
the float64 oracle on it, and all-reduces the parameter gradients; the result must equal the
full-batch gradients, and every per-row output must equal the matching rows of the full run."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_bwd_b200 import dp
from selective_state_space_bwd_b200 import inputs as gen


def test_shard_rows_partition():
    for B in (1, 2, 7, 8, 9):
        for W in (1, 2, 3, 4):
            spans = [dp.shard_rows(B, r, W) for r in range(W)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(spans[i][1] == spans[i + 1][0] for i in range(W - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = gen.real_inputs(5, 40, 8, 4, gen.F32, "mamba", seed=21)
        lo, hi = dp.shard_rows(5, rank, world)
        sl = slice(lo, hi)
        o = oracle.real(inp["x"][sl], inp["delta_raw"][sl], inp["A_log"], inp["Bm"][sl],
                        inp["Cm"][sl], inp["Dskip"], inp["dy"][sl], chunk=16, threads=1)
        dA = torch.from_numpy(o["dA_log"])
        dD = torch.from_numpy(o["dD"])
        dp.allreduce_param_grads(dA, dD)
        np.savez(os.path.join(result_dir, f"rank{rank}.npz"), dA=dA.numpy(), dD=dD.numpy(),
                 dx=o["dx"], dB=o["dB"], lo=lo, hi=hi)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_allreduce_matches_full_batch(tmp_path, oracle_mod):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    inp = gen.real_inputs(5, 40, 8, 4, gen.F32, "mamba", seed=21)
    full = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                           inp["Dskip"], inp["dy"], chunk=16, threads=1)
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        np.testing.assert_allclose(z["dA"], full["dA_log"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(z["dD"], full["dD"], rtol=1e-12, atol=1e-14)
        lo, hi = int(z["lo"]), int(z["hi"])
        np.testing.assert_allclose(z["dx"], full["dx"][lo:hi], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(z["dB"], full["dB"][lo:hi], rtol=1e-13, atol=1e-14)


def _worker_packed(rank, world, port, result_dir):
    """Scan and step-size projection on this rank's batch rows; every parameter gradient (dA_log,
    dD, dw, dbias) summed over the ranks in one packed all-reduce."""
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = gen.real_inputs(5, 24, 16, 4, gen.F32, "mamba", seed=31)
        pj = gen.dtproj_inputs(5, 24, 16, 16, seed=32)
        lo, hi = dp.shard_rows(5, rank, world)
        sl = slice(lo, hi)
        o = oracle.real(inp["x"][sl], inp["delta_raw"][sl], inp["A_log"], inp["Bm"][sl],
                        inp["Cm"][sl], inp["Dskip"], inp["dy"][sl], chunk=16, threads=1)
        q = oracle.dtproj(pj["u"][sl], pj["w"], pj["bias"], pj["g"][sl])
        grads = [torch.from_numpy(np.ascontiguousarray(a)) for a in (o["dA_log"], o["dD"], q["dw"], q["dbias"])]
        dp.allreduce_grads(grads)
        np.savez(os.path.join(result_dir, f"packed{rank}.npz"), *[g.numpy() for g in grads])
    finally:
        dist.destroy_process_group()


def test_two_rank_packed_allreduce_of_scan_and_projection_grads(tmp_path, oracle_mod):
    world = 2
    mp.spawn(_worker_packed, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    inp = gen.real_inputs(5, 24, 16, 4, gen.F32, "mamba", seed=31)
    pj = gen.dtproj_inputs(5, 24, 16, 16, seed=32)
    full = oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                           inp["Dskip"], inp["dy"], chunk=16, threads=1)
    fq = oracle_mod.dtproj(pj["u"], pj["w"], pj["bias"], pj["g"])
    want = (full["dA_log"], full["dD"], fq["dw"], fq["dbias"])
    for r in range(world):
        z = np.load(tmp_path / f"packed{r}.npz")
        for i, ref in enumerate(want):
            np.testing.assert_allclose(z[f"arr_{i}"], ref, rtol=1e-12, atol=1e-12)
