"""GPU-vs-oracle parity of the real-mode options, called through ssm_scan_fwd_ex / ssm_scan_bwd_ex:
zero-order-hold input term, initial state h0, final state hL, upstream gradient dhL and dh0.

Tolerances as for the plain calls (relative L2 per output tensor): fp32 I/O forward outputs
(y, hL, checkpoints) <= 1e-5 and gradients (dh0 included) <= 1e-4; bf16 I/O <= 2e-2.  Also checks
that streaming a sequence through two calls (hL of the first as h0 of the second, dh0 of the
second as dhL of the first) reproduces one call, and the empty sequence."""

import numpy as np
import pytest
import torch

from selective_state_space_bwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu

FWD_TOL_F32, GRAD_TOL_F32, TOL_BF16 = 1e-5, 1e-4, 2e-2
GRADS = ("dx", "ddelta_raw", "dA_log", "dB", "dC", "dD", "dh0")


@pytest.fixture(scope="module")
def S():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from selective_state_space_bwd_b200 import build, ssm_scan
    build.build()
    ssm_scan.lib()
    return ssm_scan


def rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = np.linalg.norm(b.ravel())
    num = np.linalg.norm((a - b).ravel())
    return num / den if den > 0 else num


def _inputs(B, L, D, N, io, kind, seed):
    inp = gen.real_inputs(B, L, D, N, io, kind, seed)
    rng = np.random.default_rng(seed + 500)
    inp["h0"] = rng.standard_normal((B, D, N)).astype(np.float32)
    inp["dhL"] = rng.standard_normal((B, D, N)).astype(np.float32)
    return inp


def _dev(inp, io):
    dt = torch.bfloat16 if io == gen.BF16 else torch.float32
    f32 = ("A_log", "Dskip", "h0", "dhL")
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to("cuda", torch.float32 if k in f32 else dt)
            for k, v in inp.items()}


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def run_gpu(S, d, zoh, T, seg_chunks=0, h0=True, dhL=True):
    y, ckpt, hL = S.ssm_scan_fwd_ex(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"],
                                    d["Dskip"], zoh=zoh, h0=d["h0"] if h0 else None, chunk=T,
                                    seg_chunks=seg_chunks)
    g = S.ssm_scan_bwd_ex(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"], ckpt,
                          d["dy"], zoh=zoh, h0=d["h0"] if h0 else None,
                          dhL=d["dhL"] if dhL else None, chunk=T, seg_chunks=seg_chunks)
    torch.cuda.synchronize()
    out = {"y": _np(y), "ckpt": _np(ckpt), "hL": _np(hL)}
    out.update({k: _np(v) for k, v in g.items()})
    return out


def run_oracle(oracle_mod, inp, zoh, T, h0=True, dhL=True):
    return oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                           inp["Dskip"], inp["dy"], chunk=T, want_ckpt=True, zoh=zoh,
                           h0=inp["h0"] if h0 else None, dhL=inp["dhL"] if dhL else None)


def check(got, ref, io):
    tf = TOL_BF16 if io == gen.BF16 else FWD_TOL_F32
    tg = TOL_BF16 if io == gen.BF16 else GRAD_TOL_F32
    errs = {k: rel_l2(got[k], ref[k]) for k in ("y", "ckpt", "hL") + GRADS}
    bad = {k: e for k, e in errs.items() if e > (tf if k in ("y", "ckpt", "hL") else tg)}
    assert not bad, (bad, errs)


CASES = [
    # B, L, D, N, T, io, kind, seg_chunks
    (2, 300, 64, 16, 64, gen.F32, "mamba", 0),
    (2, 300, 64, 16, 64, gen.F32, "mamba", 2),     # forced time segments (summary + carry)
    (1, 257, 32, 8, 32, gen.F32, "stiff", 3),
    (3, 129, 40, 4, 16, gen.F32, "mamba", 0),
    (2, 520, 96, 16, 128, gen.BF16, "mamba", 0),
    (1, 1000, 64, 16, 128, gen.F32, "stiff", 0),
    # more than 444 CTAs of 32 channels: the backward instance for four CTAs per SM
    (15, 200, 1024, 16, 64, gen.F32, "stiff", 0),
    (4, 260, 4096, 16, 128, gen.BF16, "mamba", 0),
]


@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("B,L,D,N,T,io,kind,seg", CASES)
def test_options_parity(S, oracle_mod, zoh, B, L, D, N, T, io, kind, seg):
    inp = _inputs(B, L, D, N, io, kind, seed=B * 1000 + L + N)
    got = run_gpu(S, _dev(inp, io), zoh, T, seg)
    ref = run_oracle(oracle_mod, inp, zoh, T)
    check(got, ref, io)


@pytest.mark.parametrize("zoh", [False, True])
def test_zoh_without_state_matches_oracle(S, oracle_mod, zoh):
    inp = _inputs(2, 333, 64, 16, gen.F32, "mamba", seed=77)
    got = run_gpu(S, _dev(inp, gen.F32), zoh, 128, h0=False, dhL=False)
    ref = run_oracle(oracle_mod, inp, zoh, 128, h0=False, dhL=False)
    check(got, ref, gen.F32)


def test_defaults_equal_plain_calls_bitwise(S):
    inp = _inputs(2, 300, 64, 16, gen.F32, "mamba", seed=5)
    d = _dev(inp, gen.F32)
    y0, ck0 = S.ssm_scan_fwd(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"], chunk=64)
    g0 = S.ssm_scan_bwd(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"], ck0, d["dy"], chunk=64)
    got = run_gpu(S, d, False, 64, h0=False, dhL=False)
    assert np.array_equal(_np(y0), got["y"])
    for k, v in g0.items():
        assert np.array_equal(_np(v), got[k]), k
    np.testing.assert_array_equal(got["hL"], _np(ck0)[:, -1])


@pytest.mark.parametrize("zoh", [False, True])
def test_streaming_two_calls_equals_one(S, zoh):
    """hL of the first half feeds h0 of the second; dh0 of the second half feeds dhL of the first."""
    B, L, D, N, T, L1 = 2, 512, 64, 16, 128, 256
    inp = _inputs(B, L, D, N, gen.F32, "mamba", seed=31)
    d = _dev(inp, gen.F32)
    full = run_gpu(S, d, zoh, T)
    first = {k: (v[:, :L1].contiguous() if v.dim() == 3 and v.shape[1] == L else v) for k, v in d.items()}
    second = {k: (v[:, L1:].contiguous() if v.dim() == 3 and v.shape[1] == L else v) for k, v in d.items()}
    y1, ck1, hL1 = S.ssm_scan_fwd_ex(first["x"], first["delta_raw"], d["A_log"], first["Bm"],
                                     first["Cm"], d["Dskip"], zoh=zoh, h0=d["h0"], chunk=T)
    y2, ck2, hL2 = S.ssm_scan_fwd_ex(second["x"], second["delta_raw"], d["A_log"], second["Bm"],
                                     second["Cm"], d["Dskip"], zoh=zoh, h0=hL1, chunk=T)
    g2 = S.ssm_scan_bwd_ex(second["x"], second["delta_raw"], d["A_log"], second["Bm"],
                           second["Cm"], d["Dskip"], ck2, second["dy"], zoh=zoh, h0=hL1,
                           dhL=d["dhL"], chunk=T)
    g1 = S.ssm_scan_bwd_ex(first["x"], first["delta_raw"], d["A_log"], first["Bm"], first["Cm"],
                           d["Dskip"], ck1, first["dy"], zoh=zoh, h0=d["h0"], dhL=g2["dh0"],
                           chunk=T)
    torch.cuda.synchronize()
    y = np.concatenate([_np(y1), _np(y2)], axis=1)
    assert rel_l2(y, full["y"]) <= FWD_TOL_F32
    assert rel_l2(_np(hL2), full["hL"]) <= FWD_TOL_F32
    for k in ("dx", "ddelta_raw", "dB", "dC"):
        got = np.concatenate([_np(g1[k]), _np(g2[k])], axis=1)
        assert rel_l2(got, full[k]) <= GRAD_TOL_F32, k
    for k in ("dA_log", "dD"):
        assert rel_l2(_np(g1[k]) + _np(g2[k]), full[k]) <= GRAD_TOL_F32, k
    assert rel_l2(_np(g1["dh0"]), full["dh0"]) <= GRAD_TOL_F32


def test_empty_sequence_passes_the_state_through(S):
    inp = _inputs(2, 0, 32, 16, gen.F32, "mamba", seed=3)
    got = run_gpu(S, _dev(inp, gen.F32), True, 64)
    np.testing.assert_array_equal(got["hL"], inp["h0"])
    np.testing.assert_array_equal(got["dh0"], inp["dhL"])
    assert not got["dA_log"].any() and not got["dD"].any()


FUSED_CASES = [
    # B, L, D, N, T, io, kind, seg_chunks: backward launches whose CTAs all fit at once
    (2, 300, 64, 16, 64, gen.F32, "mamba", 0),
    (2, 300, 64, 16, 64, gen.F32, "mamba", 2),     # time segments (summary + carry)
    (3, 517, 72, 8, 32, gen.F32, "stiff", 0),
    (2, 129, 136, 4, 16, gen.BF16, "mamba", 0),
    (4, 700, 1024, 16, 128, gen.BF16, "mamba", 0),  # 128 CTAs, 6 chunks
    (15, 200, 1024, 16, 64, gen.F32, "stiff", 0),  # 480 CTAs: the four-CTA-per-SM instance
]


@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("B,L,D,N,T,io,kind,seg", FUSED_CASES)
def test_fused_sums_parity(S, oracle_mod, zoh, B, L, D, N, T, io, kind, seg):
    """SSM_FUSED_SUMS: dB and dC summed inside the scan kernel (cooperative launches) against the
    oracle; the other gradients bitwise equal to the call without the flag; the status clean; a
    second call bitwise equal (a fixed order of the channel tiles)."""
    inp = _inputs(B, L, D, N, io, kind, seed=B * 7 + L + N)
    d = _dev(inp, io)
    y, ckpt, hL = S.ssm_scan_fwd_ex(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"],
                                    d["Dskip"], zoh=zoh, h0=d["h0"], chunk=T, seg_chunks=seg)
    args = (d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"], ckpt, d["dy"])
    shape = S.real_shape(B, L, D, N, T, S._io_of(d["x"]), seg)
    ws = torch.empty(S.workspace_bytes(shape, True), dtype=torch.uint8, device="cuda")
    g1 = S.ssm_scan_bwd_ex(*args, zoh=zoh, h0=d["h0"], dhL=d["dhL"], chunk=T, seg_chunks=seg,
                           ws=ws, fused_sums=True)
    g1 = {k: v.clone() for k, v in g1.items()}
    assert S.ssm_scan_status(ws) == 0
    g2 = S.ssm_scan_bwd_ex(*args, zoh=zoh, h0=d["h0"], dhL=d["dhL"], chunk=T, seg_chunks=seg,
                           ws=ws, fused_sums=True)
    plain = S.ssm_scan_bwd_ex(*args, zoh=zoh, h0=d["h0"], dhL=d["dhL"], chunk=T, seg_chunks=seg)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k
        if k not in ("dB", "dC"):
            assert torch.equal(g1[k], plain[k]), k
    got = {"y": _np(y), "ckpt": _np(ckpt), "hL": _np(hL)}
    got.update({k: _np(v) for k, v in g1.items()})
    check(got, run_oracle(oracle_mod, inp, zoh, T), io)
