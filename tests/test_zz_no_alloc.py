"""The allocation-free forward entry point, ssm_scan_fwd_noalloc.

It serves callers that cannot allocate device memory themselves (for instance a plugin whose host
framework owns all device memory, or a loop that must never call cudaMalloc): its scratch is an
8 MiB array built into the library instead of a caller-provided workspace.  These tests call it
through the C ABI twice in a row.  It runs the same kernels with the same launch plan as the
regular ssm_scan_fwd (the built-in array only stands in for the workspace), and the forward has
no atomics, so its outputs must equal the regular forward's bit for bit; one fp32 case is also
checked against the float64 oracle directly.  This file is collected last on purpose, and passes
both alone in a fresh process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

from selective_state_space_bwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from selective_state_space_bwd_b200 import build, ssm_scan
    build.build()
    ssm_scan.lib()
    return ssm_scan


def _rel(a, b):
    a = a.detach().double().cpu().numpy() if torch.is_tensor(a) else np.asarray(a, np.float64)
    b = b.detach().double().cpu().numpy() if torch.is_tensor(b) else np.asarray(b, np.float64)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def _inputs(B, L, D, N, io, seed):
    dt = torch.bfloat16 if io == gen.BF16 else torch.float32
    inp = gen.real_inputs(B, L, D, N, io, "mamba", seed=seed)
    t = {k: torch.from_numpy(v).cuda().to(dt if k not in ("A_log", "Dskip") else torch.float32)
         for k, v in inp.items()}
    return inp, t


@pytest.mark.parametrize("B,L,D,N,T,io,sc", [
    (1, 4096, 64, 16, 128, gen.F32, 0),    # few CTAs: split into time segments (scratch in use)
    (2, 300, 40, 16, 128, gen.BF16, 0),    # one segment: scratch holds only the status word
    (3, 517, 72, 8, 32, gen.F32, 2),
])
def test_noalloc_forward_equals_regular_forward(S, B, L, D, N, T, io, sc):
    _, t = _inputs(B, L, D, N, io, L + D)
    args = (t["x"], t["delta_raw"], t["A_log"], t["Bm"], t["Cm"], t["Dskip"])
    y_ref, ck_ref = S.ssm_scan_fwd(*args, chunk=T, seg_chunks=sc)
    torch.cuda.synchronize()
    for call in range(2):  # two calls in a row share the built-in scratch
        y = torch.full_like(y_ref, float("nan"))
        ck = torch.full_like(ck_ref, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        S.ssm_scan_fwd_noalloc(*args, y, ck, chunk=T, seg_chunks=sc)
        torch.cuda.synchronize()
        if call == 1:  # after the first call's one-time address lookup, nothing is allocated
            assert torch.cuda.mem_get_info()[0] == free_before
        assert torch.equal(y, y_ref), f"call {call}: y differs from ssm_scan_fwd"
        assert torch.equal(ck, ck_ref), f"call {call}: checkpoints differ from ssm_scan_fwd"


def test_noalloc_forward_against_oracle(S):
    # fp32, split into time segments (the built-in scratch holds summaries and entering states)
    import oracle
    B, L, D, N, T = 1, 3000, 48, 16, 64
    inp, t = _inputs(B, L, D, N, gen.F32, 7)
    ref = oracle.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                      inp["Dskip"], chunk=T, want_ckpt=True)
    y = torch.empty_like(t["x"])
    ck = torch.empty((B, -(-L // T), D, N), device="cuda")
    for _ in range(2):
        y.fill_(float("nan"))
        ck.fill_(float("nan"))
        S.ssm_scan_fwd_noalloc(t["x"], t["delta_raw"], t["A_log"], t["Bm"], t["Cm"], t["Dskip"],
                               y, ck, chunk=T)
        torch.cuda.synchronize()
        assert _rel(y, ref["y"]) <= 1e-5
        assert _rel(ck, ref["ckpt"]) <= 1e-5


def test_noalloc_rejects_problems_beyond_its_scratch(S):
    # 1024 one-chunk time segments of 1024 x 16 states need ~200 MB of scratch > 8 MiB
    B, L, D, N, T = 1, 16384, 1024, 16, 16
    shape = S.real_shape(B, L, D, N, T, S.SSM_F32, seg_chunks=1)
    assert S.workspace_bytes(shape, False) > (8 << 20)
    x = torch.zeros((B, L, D), device="cuda")
    A_log = torch.zeros((D, N), device="cuda")
    Bm = torch.zeros((B, L, N), device="cuda")
    Dskip = torch.zeros(D, device="cuda")
    y = torch.empty_like(x)
    ck = torch.empty((B, L // T, D, N), device="cuda")
    with pytest.raises(S.SsmError) as e:
        S.ssm_scan_fwd_noalloc(x, x, A_log, Bm, Bm, Dskip, y, ck, chunk=T, seg_chunks=1)
    assert e.value.code == 4
