"""GPU parity of the step-size projection (ssm_dtproj_fwd / ssm_dtproj_bwd) against the float64
oracle, on the same bf16 operands.  Tolerances (relative L2): delta_raw and du, rounded to bf16
once, 4e-3 (bf16 keeps 8 significant bits: relative rounding error below 2^-9, about 1e-3 in the
L2 norm); dw and dbias, fp32 sums of up to 65536 products accumulated in fp32, 1e-4; the whole
pipeline (projection, scan, projection backward) at the bf16 I/O tolerance 2e-2."""

import numpy as np
import pytest
import torch

from selective_state_space_bwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu

BF16_TOL, F32_TOL = 4e-3, 1e-4


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


def bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


@pytest.mark.parametrize("B,L,D,R", [(1, 300, 40, 16), (2, 500, 1536, 48), (1, 129, 8, 256),
                                     (3, 7, 64, 32), (1, 4096, 4096, 128), (8, 2048, 1536, 48),
                                     (2, 333, 200, 64), (1, 1000, 264, 80), (2, 1000, 520, 192)])
def test_dtproj_matches_oracle(S, oracle_mod, B, L, D, R):
    p = gen.dtproj_inputs(B, L, D, R, seed=B + L + D + R)
    u, w, g = bf(p["u"]), bf(p["w"]), bf(p["g"])
    bias = torch.from_numpy(p["bias"]).cuda()
    dr = S.ssm_dtproj_fwd(u, w, bias)
    out = S.ssm_dtproj_bwd(u, w, g)
    torch.cuda.synchronize()
    ref = oracle_mod.dtproj(p["u"], p["w"], p["bias"], p["g"])
    assert rel(dr.float().cpu().numpy(), ref["delta_raw"]) <= BF16_TOL
    assert rel(out["du"].float().cpu().numpy(), ref["du"]) <= BF16_TOL
    assert rel(out["dw"].cpu().numpy(), ref["dw"]) <= F32_TOL
    assert rel(out["dbias"].cpu().numpy(), ref["dbias"]) <= F32_TOL


def test_dtproj_no_bias_and_empty(S):
    p = gen.dtproj_inputs(1, 64, 32, 16, seed=1)
    u, w = bf(p["u"]), bf(p["w"])
    a = S.ssm_dtproj_fwd(u, w, None)
    b = S.ssm_dtproj_fwd(u, w, torch.zeros(32, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    e = gen.dtproj_inputs(2, 0, 32, 16, seed=2)
    out = S.ssm_dtproj_bwd(bf(e["u"]), bf(e["w"]), bf(e["g"]))
    torch.cuda.synchronize()
    assert not out["dw"].any() and not out["dbias"].any()


def test_dtproj_deterministic(S):
    p = gen.dtproj_inputs(2, 1500, 256, 64, seed=3)
    u, w, g = bf(p["u"]), bf(p["w"]), bf(p["g"])
    r1 = S.ssm_dtproj_bwd(u, w, g)
    r2 = S.ssm_dtproj_bwd(u, w, g)
    torch.cuda.synchronize()
    for k in r1:
        assert torch.equal(r1[k], r2[k]), k


def test_projection_scan_pipeline(S, oracle_mod):
    """u -> delta_raw (projection) -> scan fwd + bwd -> du, dw, dbias (projection backward),
    all on the GPU, against the oracle's chain on the GPU's bf16 operands."""
    B, L, D, N, R = 2, 300, 64, 16, 32
    c = gen.real_inputs(B, L, D, N, gen.BF16, "mamba", seed=5)
    p = gen.dtproj_inputs(B, L, D, R, seed=6)
    d = {k: (bf(v) if k in ("x", "Bm", "Cm", "dy") else torch.from_numpy(v).cuda())
         for k, v in c.items() if k != "delta_raw"}
    u, w = bf(p["u"]), bf(p["w"])
    bias = torch.from_numpy(p["bias"]).cuda()
    dr = S.ssm_dtproj_fwd(u, w, bias)
    y, ck = S.ssm_scan_fwd(d["x"], dr, d["A_log"], d["Bm"], d["Cm"], d["Dskip"], chunk=64)
    gs = S.ssm_scan_bwd(d["x"], dr, d["A_log"], d["Bm"], d["Cm"], d["Dskip"], ck, d["dy"], chunk=64)
    pg = S.ssm_dtproj_bwd(u, w, gs["ddelta_raw"])
    torch.cuda.synchronize()
    ref_dr = oracle_mod.dtproj(p["u"], p["w"], p["bias"])["delta_raw"]
    sc = oracle_mod.real(c["x"], ref_dr, c["A_log"], c["Bm"], c["Cm"], c["Dskip"], c["dy"], chunk=64)
    ref = oracle_mod.dtproj(p["u"], p["w"], p["bias"], sc["ddelta_raw"])
    assert rel(y.float().cpu().numpy(), sc["y"]) <= 2e-2
    for k in ("du", "dw", "dbias"):
        assert rel(pg[k].float().cpu().numpy(), ref[k]) <= 2e-2, k


def test_dtproj_status_clean(S):
    """No bounded tensor-core wait of the projection kernels gives up: the workspace status word
    reads SSM_OK after each call."""
    p = gen.dtproj_inputs(2, 700, 320, 64, seed=11)
    u, w, g = bf(p["u"]), bf(p["w"]), bf(p["g"])
    shp = S.dtproj_shape(2 * 700, 320, 64)
    wsf = torch.full((S.dtproj_workspace_bytes(shp, False),), 0xFF, dtype=torch.uint8, device="cuda")
    wsb = torch.full((S.dtproj_workspace_bytes(shp, True),), 0xFF, dtype=torch.uint8, device="cuda")
    S.ssm_dtproj_fwd(u, w, torch.from_numpy(p["bias"]).cuda(), ws=wsf)
    assert S.ssm_scan_status(wsf) == S.SSM_OK  # the call reset the word, no wait gave up
    S.ssm_dtproj_bwd(u, w, g, ws=wsb)
    assert S.ssm_scan_status(wsb) == S.SSM_OK
