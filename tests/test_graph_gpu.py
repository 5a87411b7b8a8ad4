"""The library's calls can be captured in a CUDA graph: a captured forward + backward (real mode;
complex mode; Flash PD-SSM; the step-size projection) replayed on new inputs copied into the
captured buffers gives bitwise the outputs of eager calls."""

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


@pytest.mark.parametrize("fused", [False, True])
def test_captured_fwd_bwd_replays_bitwise(S, fused):
    """fused: the backward with SSM_FUSED_SUMS (cooperative launches and the chunk counters'
    memset in the graph)."""
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
        if fused:
            S.ssm_scan_bwd_ex(a["x"], a["delta_raw"], a["A_log"], a["Bm"], a["Cm"], a["Dskip"], ck,
                              a["dy"], chunk=T, out=out, ws=wsb, fused_sums=True)
        else:
            S.ssm_scan_bwd(a["x"], a["delta_raw"], a["A_log"], a["Bm"], a["Cm"], a["Dskip"], ck,
                           a["dy"], chunk=T, out=out, ws=wsb)

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
    if fused:
        ref = S.ssm_scan_bwd_ex(b["x"], b["delta_raw"], b["A_log"], b["Bm"], b["Cm"], b["Dskip"], ck2,
                                b["dy"], chunk=T, fused_sums=True)
    else:
        ref = S.ssm_scan_bwd(b["x"], b["delta_raw"], b["A_log"], b["Bm"], b["Cm"], b["Dskip"], ck2,
                             b["dy"], chunk=T)
    torch.cuda.synchronize()
    assert torch.equal(got["y"], y2)
    for k, v in ref.items():
        if k in out:
            assert torch.equal(got[k], v), k
    assert S.ssm_scan_status(wsb) == 0


def _capture_and_replay(step, bufs, fresh):
    """Warm up `step` eagerly, capture it, copy `fresh` into the captured input buffers `bufs`,
    replay; returns nothing (the outputs live in the captured buffers)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for k in bufs:
        bufs[k].copy_(fresh[k])
    g.replay()
    torch.cuda.synchronize()
    return g


def test_captured_complex_and_pdssm_and_projection_replay_bitwise(S):
    # complex mode (warp-specialised kernels with named barriers)
    c1, c2 = gen.complex_inputs(2, 300, 128, seed=1), gen.complex_inputs(2, 300, 128, seed=2)
    a = {k: torch.from_numpy(v).cuda() for k, v in c1.items()}
    h = torch.empty_like(a["u"])
    outc = dict(du=torch.empty_like(a["g"]), dr=torch.empty_like(a["r"]), dphi=torch.empty_like(a["phi"]),
                dlambda=torch.empty_like(a["lam"]), domega=torch.empty_like(a["omega"]))

    def cstep():
        S.ssm_scan_complex_fwd(a["u"], a["r"], a["phi"], a["lam"], a["omega"], h=h)
        S.ssm_scan_complex_bwd_traj(h, a["r"], a["phi"], a["lam"], a["omega"], a["g"], out=outc)

    _capture_and_replay(cstep, a, {k: torch.from_numpy(v).cuda() for k, v in c2.items()})
    got = {"h": h.clone(), **{k: v.clone() for k, v in outc.items()}}
    b = {k: torch.from_numpy(v).cuda() for k, v in c2.items()}
    h2 = S.ssm_scan_complex_fwd(b["u"], b["r"], b["phi"], b["lam"], b["omega"])
    o2 = S.ssm_scan_complex_bwd_traj(h2, b["r"], b["phi"], b["lam"], b["omega"], b["g"])
    torch.cuda.synchronize()
    assert torch.equal(got["h"], h2)
    for k in o2:
        assert torch.equal(got[k], o2[k]), k

    # complex mode from checkpoints (forward writing checkpoints, checkpointed backward)
    ck = torch.empty((2, -(-300 // 128), 128), dtype=torch.complex64, device="cuda")
    outk = {k: torch.empty_like(v) for k, v in outc.items()}

    def kstep():
        S.ssm_scan_complex_fwd(a["u"], a["r"], a["phi"], a["lam"], a["omega"], h=h, ckpt=ck)
        S.ssm_scan_complex_bwd(a["u"], a["r"], a["phi"], a["lam"], a["omega"], ck, a["g"], out=outk)

    _capture_and_replay(kstep, a, {k: torch.from_numpy(v).cuda() for k, v in c1.items()})
    b1 = {k: torch.from_numpy(v).cuda() for k, v in c1.items()}
    _, ck1 = S.ssm_scan_complex_fwd(b1["u"], b1["r"], b1["phi"], b1["lam"], b1["omega"], want_ckpt=True)
    o1 = S.ssm_scan_complex_bwd(b1["u"], b1["r"], b1["phi"], b1["lam"], b1["omega"], ck1, b1["g"])
    torch.cuda.synchronize()
    assert torch.equal(ck, ck1)
    for k in o1:
        assert torch.equal(outk[k], o1[k]), k

    # Flash PD-SSM (fused argmax / score gradient, warp-specialised backward)
    p1, p2 = gen.pdssm_inputs(2, 400, 32, 16, 8, seed=1), gen.pdssm_inputs(2, 400, 32, 16, 8, seed=2)
    q = {k: torch.from_numpy(v).cuda() for k, v in p1.items()}
    hp = torch.empty_like(q["d"])
    sel = torch.empty(q["scores"].shape[:3], dtype=torch.int32, device="cuda")
    outp = dict(dd=torch.empty_like(q["d"]), dbt=torch.empty_like(q["d"]),
                dscores=torch.empty_like(q["scores"]), dh0=torch.empty_like(q["h0"]))

    def pstep():
        S.ssm_pdssm_fwd(q["scores"], q["dictionary"], q["d"], q["bt"], h0=q["h0"], h=hp, sel=sel)
        S.ssm_pdssm_bwd(q["scores"], q["dictionary"], q["d"], hp, sel, q["g"], tau=0.5, h0=q["h0"],
                        out=outp)

    _capture_and_replay(pstep, q, {k: torch.from_numpy(v).cuda() for k, v in p2.items()})
    got = {"h": hp.clone(), "sel": sel.clone(), **{k: v.clone() for k, v in outp.items()}}
    r = {k: torch.from_numpy(v).cuda() for k, v in p2.items()}
    h3, s3 = S.ssm_pdssm_fwd(r["scores"], r["dictionary"], r["d"], r["bt"], h0=r["h0"])
    o3 = S.ssm_pdssm_bwd(r["scores"], r["dictionary"], r["d"], h3, s3, r["g"], tau=0.5, h0=r["h0"])
    torch.cuda.synchronize()
    assert torch.equal(got["h"], h3) and torch.equal(got["sel"], s3)
    for k in o3:
        assert torch.equal(got[k], o3[k]), k

    # step-size projection
    j1, j2 = gen.dtproj_inputs(2, 700, 256, 48, seed=1), gen.dtproj_inputs(2, 700, 256, 48, seed=2)
    bfk = ("u", "w", "g")
    t = {k: torch.from_numpy(v).cuda().to(torch.bfloat16 if k in bfk else torch.float32)
         for k, v in j1.items()}
    dr = torch.empty((2, 700, 256), dtype=torch.bfloat16, device="cuda")
    outj = dict(du=torch.empty_like(t["u"]), dw=torch.empty((256, 48), device="cuda"),
                dbias=torch.empty(256, device="cuda"))

    def jstep():
        S.ssm_dtproj_fwd(t["u"], t["w"], t["bias"], delta_raw=dr)
        S.ssm_dtproj_bwd(t["u"], t["w"], t["g"], out=outj)

    _capture_and_replay(jstep, t, {k: torch.from_numpy(v).cuda().to(torch.bfloat16 if k in bfk else torch.float32)
                                   for k, v in j2.items()})
    got = {"dr": dr.clone(), **{k: v.clone() for k, v in outj.items()}}
    u = {k: torch.from_numpy(v).cuda().to(torch.bfloat16 if k in bfk else torch.float32) for k, v in j2.items()}
    dr2 = S.ssm_dtproj_fwd(u["u"], u["w"], u["bias"])
    o4 = S.ssm_dtproj_bwd(u["u"], u["w"], u["g"])
    torch.cuda.synchronize()
    assert torch.equal(got["dr"], dr2)
    for k in o4:
        assert torch.equal(got[k], o4[k]), k
