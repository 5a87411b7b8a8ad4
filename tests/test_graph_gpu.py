"""The scan calls can be captured in a CUDA graph: a captured forward + backward replayed on new
inputs (copied into the captured buffers) gives bitwise the outputs of eager calls."""

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


def _dev(inp):
    return {k: torch.from_numpy(v).cuda().to(torch.bfloat16 if k not in ("A_log", "Dskip") else torch.float32)
            for k, v in inp.items()}


def test_captured_fwd_bwd_replays_bitwise(S):
    B, L, D, N, T = 2, 1000, 128, 16, 128
    a = _dev(gen.real_inputs(B, L, D, N, gen.BF16, "mamba", seed=1))
    shape = S.real_shape(B, L, D, N, T, S.SSM_BF16)
    wsf = torch.empty(S.workspace_bytes(shape, False), dtype=torch.uint8, device="cuda")
    wsb = torch.empty(S.workspace_bytes(shape, True), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(a["x"])
    ck = torch.empty((B, -(-L // T), D, N), dtype=torch.float32, device="cuda")
    out = dict(dx=torch.empty_like(a["x"]), ddelta_raw=torch.empty_like(a["x"]),
               dA_log=torch.empty_like(a["A_log"]), dB=torch.empty_like(a["Bm"]),
               dC=torch.empty_like(a["Cm"]), dD=torch.empty_like(a["Dskip"]))

    def step():
        S.ssm_scan_fwd(a["x"], a["delta_raw"], a["A_log"], a["Bm"], a["Cm"], a["Dskip"], chunk=T,
                       y=y, ckpt=ck, ws=wsf)
        S.ssm_scan_bwd(a["x"], a["delta_raw"], a["A_log"], a["Bm"], a["Cm"], a["Dskip"], ck, a["dy"],
                       chunk=T, out=out, ws=wsb)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm-up outside the capture (kernel attributes are set on first use)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    # new inputs into the captured buffers, replay, and compare with eager calls
    b = _dev(gen.real_inputs(B, L, D, N, gen.BF16, "mamba", seed=2))
    for k in a:
        a[k].copy_(b[k])
    g.replay()
    torch.cuda.synchronize()
    got = {"y": y.clone(), **{k: v.clone() for k, v in out.items()}}
    y2, ck2 = S.ssm_scan_fwd(b["x"], b["delta_raw"], b["A_log"], b["Bm"], b["Cm"], b["Dskip"], chunk=T)
    ref = S.ssm_scan_bwd(b["x"], b["delta_raw"], b["A_log"], b["Bm"], b["Cm"], b["Dskip"], ck2, b["dy"],
                         chunk=T)
    torch.cuda.synchronize()
    assert torch.equal(got["y"], y2)
    for k, v in ref.items():
        assert torch.equal(got[k], v), k
    assert S.ssm_scan_status(wsb) == 0
