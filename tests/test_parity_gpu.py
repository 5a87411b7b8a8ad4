"""GPU-vs-oracle parity for the real and complex scans, called through the C ABI.

Tolerances (relative L2 per output tensor, over the whole tensor, in float64):
  fp32 / complex64 I/O: forward outputs <= 1e-5, gradients <= 1e-4;
  bf16 I/O:             every output   <= 2e-2.
Both sides consume the same seeded inputs (bf16 workloads are drawn already bf16-rounded).

Full-size workloads run in exactly the launch configuration the bench times and are checked on
sampled channels the oracle computes one by one: the upstream gradient is zeroed outside a channel
subset, so the cross-channel sums (dB, dC; dr, dphi) cover only channels the oracle also sums, and
every other gradient row must come out exactly zero.  The unmasked run is checked with the Euler
homogeneity identities, which hold at any size.
"""

import math

import numpy as np
import pytest
import torch

from selective_state_space_bwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu

FWD_TOL_F32, GRAD_TOL_F32, TOL_BF16 = 1e-5, 1e-4, 2e-2


@pytest.fixture(scope="module")
def S():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from selective_state_space_bwd_b200 import build, ssm_scan
    build.build()
    ssm_scan.lib()
    return ssm_scan


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.complex128 if np.iscomplexobj(a) or np.iscomplexobj(b) else np.float64)
    b = np.asarray(b, dtype=a.dtype)
    den = np.linalg.norm(b.ravel())
    num = np.linalg.norm((a - b).ravel())
    return num / den if den > 0 else num


def to_dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def np64(t):
    return t.detach().to(torch.float64 if not t.is_complex() else torch.complex128).cpu().numpy()


def run_real(S, inp, io, T, seg_chunks=0):
    dt = torch.bfloat16 if io == gen.BF16 else torch.float32
    x, dr, dy = (to_dev(inp[k], dt) for k in ("x", "delta_raw", "dy"))
    Bm, Cm = to_dev(inp["Bm"], dt), to_dev(inp["Cm"], dt)
    A_log, Dskip = to_dev(inp["A_log"], torch.float32), to_dev(inp["Dskip"], torch.float32)
    y, ckpt = S.ssm_scan_fwd(x, dr, A_log, Bm, Cm, Dskip, chunk=T, seg_chunks=seg_chunks)
    g = S.ssm_scan_bwd(x, dr, A_log, Bm, Cm, Dskip, ckpt, dy, chunk=T, seg_chunks=seg_chunks)
    torch.cuda.synchronize()
    out = {"y": np64(y), "ckpt": np64(ckpt)}
    out.update({k: np64(v) for k, v in g.items()})
    return out


def run_oracle(oracle_mod, inp, T, d_range=None):
    return oracle_mod.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                           inp["Dskip"], inp["dy"], chunk=T, d_range=d_range, want_ckpt=True)


GRADS = ("dx", "ddelta_raw", "dA_log", "dB", "dC", "dD")


def check_real(got, ref, io, sel=None):
    """Compare every output; ``sel`` restricts per-channel outputs to a channel subset."""
    tf = TOL_BF16 if io == gen.BF16 else FWD_TOL_F32
    tg = TOL_BF16 if io == gen.BF16 else GRAD_TOL_F32
    errs = {}
    for k in ("y", "ckpt") + GRADS:
        a, b = got[k], ref[k]
        if sel is not None:
            if k in ("y", "dx", "ddelta_raw"):
                a, b = a[..., sel], b[..., sel]
            elif k == "ckpt":
                a, b = a[:, :, sel], b[:, :, sel]
            elif k in ("dA_log", "dD"):
                a, b = a[sel], b[sel]
        errs[k] = rel_l2(a, b)
    for k, e in errs.items():
        tol = tf if k in ("y", "ckpt") else tg
        assert e <= tol, f"{k}: rel-L2 {e:.3e} > {tol:.1e} (all: " + \
            ", ".join(f"{kk}={v:.2e}" for kk, v in errs.items()) + ")"
    return errs


# ------------------------------------------------------------------------------ small real cases

def test_tiny_workload(S, oracle_mod):
    w = gen.WORKLOADS["tiny"]
    inp = gen.workload_inputs("tiny")
    got = run_real(S, inp, w.io, w.chunk)
    check_real(got, run_oracle(oracle_mod, inp, w.chunk), w.io)


REAL_CASES = [
    # B, L, D, N, T, io, seg_chunks
    (2, 300, 40, 16, 128, gen.F32, 0),
    (2, 300, 40, 16, 128, gen.BF16, 0),
    (1, 1000, 64, 16, 64, gen.F32, 3),
    (3, 517, 72, 8, 32, gen.F32, 2),
    (3, 517, 72, 8, 32, gen.BF16, 0),
    (2, 129, 136, 4, 16, gen.F32, 0),
    (2, 129, 136, 4, 16, gen.BF16, 5),
    (1, 700, 32, 16, 256, gen.F32, 0),
    (1, 700, 32, 16, 256, gen.BF16, 1),
    (2, 1, 32, 16, 128, gen.F32, 0),
    (2, 2, 32, 16, 16, gen.F32, 0),
    (1, 127, 32, 16, 128, gen.F32, 0),
    (1, 129, 32, 16, 128, gen.F32, 1),
    (4, 2048, 96, 16, 128, gen.BF16, 0),
    # 512 CTAs of N = 8: more than the 444 the three-CTA-per-SM instance holds at once, so the
    # backward runs as a plain launch followed by its dB/dC reduction kernel (the small cases
    # above run cooperatively, their sums fused into the scan kernel)
    (16, 150, 1024, 8, 64, gen.F32, 0),
]


@pytest.mark.parametrize("B,L,D,N,T,io,sc", REAL_CASES)
def test_real_shapes(S, oracle_mod, B, L, D, N, T, io, sc):
    inp = gen.real_inputs(B, L, D, N, io, "mamba", seed=B * 1000 + L + D)
    got = run_real(S, inp, io, T, sc)
    check_real(got, run_oracle(oracle_mod, inp, T), io)


@pytest.mark.parametrize("io", [gen.F32, gen.BF16])
def test_real_stiff_small(S, oracle_mod, io):
    inp = gen.real_inputs(1, 3000, 64, 16, io, "stiff", seed=3)
    got = run_real(S, inp, io, 128, seg_chunks=4)
    check_real(got, run_oracle(oracle_mod, inp, 128), io)


def test_chunk_size_invariance(S):
    inp = gen.real_inputs(2, 777, 64, 16, gen.F32, "mamba", seed=11)
    outs = {T: run_real(S, inp, gen.F32, T) for T in (16, 32, 64, 128, 256)}
    ref = outs[128]
    for T, o in outs.items():
        for k in ("y",) + GRADS:
            assert rel_l2(o[k], ref[k]) < 1e-5, (T, k)
    one = run_real(S, inp, gen.F32, 256, seg_chunks=1)
    for k in ("y",) + GRADS:
        assert rel_l2(one[k], outs[256][k]) < 1e-5, k


def test_deterministic(S):
    inp = gen.real_inputs(2, 640, 96, 16, gen.BF16, "mamba", seed=5)
    a = run_real(S, inp, gen.BF16, 128)
    b = run_real(S, inp, gen.BF16, 128)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_empty_sequence(S):
    x = torch.zeros((2, 0, 32), device="cuda")
    A_log = torch.zeros((32, 16), device="cuda")
    Bm = torch.zeros((2, 0, 16), device="cuda")
    Dskip = torch.ones(32, device="cuda")
    y, ck = S.ssm_scan_fwd(x, x, A_log, Bm, Bm, Dskip)
    assert y.shape == (2, 0, 32) and ck.shape == (2, 0, 32, 16)
    g = S.ssm_scan_bwd(x, x, A_log, Bm, Bm, Dskip, ck, x)
    torch.cuda.synchronize()
    assert float(g["dA_log"].abs().sum()) == 0.0 and float(g["dD"].abs().sum()) == 0.0


def test_nonfinite_status(S):
    inp = gen.real_inputs(1, 64, 32, 16, gen.F32, "mamba", seed=2)
    inp["x"][0, 10, 3] = np.inf
    dt = torch.float32
    args = [to_dev(inp[k], dt) for k in ("x", "delta_raw", "A_log", "Bm", "Cm", "Dskip")]
    shape = S.real_shape(1, 64, 32, 16, 32, S.SSM_F32)
    ws = torch.zeros(S.workspace_bytes(shape, False), dtype=torch.uint8, device="cuda")
    S.ssm_scan_fwd(*args, chunk=32, ws=ws)
    assert S.ssm_scan_status(ws) == 7
    inp["x"][0, 10, 3] = 0.0
    args[0] = to_dev(inp["x"], dt)
    S.ssm_scan_fwd(*args, chunk=32, ws=ws)
    assert S.ssm_scan_status(ws) == 0


def test_multiwave_backward_scratch_slots(S, oracle_mod):
    """A time-split backward whose launches hold more CTAs than the 592 resident ones (B=2,
    L=20000, D=1024: segments of 4 chunks x 64 CTAs, 20 segments = 1280 CTAs per launch), so
    its CTAs claim scratch slots from the workspace's slot mask.  Every output against the
    oracle, the status word clean after each call, and a second call on the same workspace
    (whose mask the first left clear) bitwise equal."""
    B, L, D, N, T = 2, 20000, 1024, 16, 128
    inp = gen.real_inputs(B, L, D, N, gen.F32, "stiff", seed=23)
    shape = S.real_shape(B, L, D, N, T, S.SSM_F32)
    assert S.kernel_launches(shape, True) == 7  # summary, carry, 2 x (scan + dB/dC sums), params
    wsb = torch.empty(S.workspace_bytes(shape, True), dtype=torch.uint8, device="cuda")
    dt = torch.float32
    x, dr, dy = (to_dev(inp[k], dt) for k in ("x", "delta_raw", "dy"))
    Bm, Cm, A_log, Dskip = (to_dev(inp[k], dt) for k in ("Bm", "Cm", "A_log", "Dskip"))
    y, ckpt = S.ssm_scan_fwd(x, dr, A_log, Bm, Cm, Dskip, chunk=T)
    g1 = S.ssm_scan_bwd(x, dr, A_log, Bm, Cm, Dskip, ckpt, dy, chunk=T, ws=wsb)
    g1 = {k: v.clone() for k, v in g1.items()}
    assert S.ssm_scan_status(wsb) == 0
    g2 = S.ssm_scan_bwd(x, dr, A_log, Bm, Cm, Dskip, ckpt, dy, chunk=T, ws=wsb)
    assert S.ssm_scan_status(wsb) == 0
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k
    got = {"y": np64(y), "ckpt": np64(ckpt)}
    got.update({k: np64(v) for k, v in g1.items()})
    check_real(got, run_oracle(oracle_mod, inp, T), gen.F32)


# ------------------------------------------------------------------------------ complex cases

def run_complex(S, c, T, seg_chunks=0, bwd="ckpt"):
    """Complex forward (trajectory and checkpoints) and one of the two backward calls: from the
    checkpoints (ssm_scan_complex_bwd) or from the stored trajectory (ssm_scan_complex_bwd_traj)."""
    u = to_dev(c["u"], torch.complex64)
    g = to_dev(c["g"], torch.complex64)
    r, phi = to_dev(c["r"], torch.float32), to_dev(c["phi"], torch.float32)
    lam, om = to_dev(c["lam"], torch.float32), to_dev(c["omega"], torch.float32)
    h, ck = S.ssm_scan_complex_fwd(u, r, phi, lam, om, chunk=T, seg_chunks=seg_chunks,
                                   want_ckpt=True)
    if bwd == "ckpt":
        gr = S.ssm_scan_complex_bwd(u, r, phi, lam, om, ck, g, chunk=T, seg_chunks=seg_chunks)
    else:
        gr = S.ssm_scan_complex_bwd_traj(h, r, phi, lam, om, g, chunk=T, seg_chunks=seg_chunks)
    torch.cuda.synchronize()
    out = {"h": np64(h), "ckpt": np64(ck)}
    out.update({k: np64(v) for k, v in gr.items()})
    return out


def check_complex_ckpt(got, T):
    """The forward's checkpoints are its own trajectory at every chunk's last step, bit for bit."""
    L = got["h"].shape[1]
    ends = [min(L, (c + 1) * T) - 1 for c in range(got["ckpt"].shape[1])]
    assert np.array_equal(got["ckpt"], got["h"][:, ends, :])


def check_complex(got, ref, sel=None):
    errs = {}
    for k in ("h", "du", "dr", "dphi", "dlambda", "domega"):
        a, b = got[k], ref[k]
        if sel is not None and k in ("h", "du"):
            a, b = a[..., sel], b[..., sel]
        elif sel is not None and k in ("dlambda", "domega"):
            a, b = a[sel], b[sel]
        errs[k] = rel_l2(a, b)
    for k, e in errs.items():
        tol = FWD_TOL_F32 if k == "h" else GRAD_TOL_F32
        assert e <= tol, f"{k}: rel-L2 {e:.3e} > {tol:.1e} ({errs})"
    return errs


@pytest.mark.parametrize("B,L,K,T,sc", [(2, 300, 64, 128, 0), (3, 517, 130, 32, 2),
                                        (1, 1000, 64, 64, 3), (2, 77, 2, 16, 0),
                                        (1, 1, 64, 128, 0), (2, 600, 200, 256, 1)])
@pytest.mark.parametrize("bwd", ["ckpt", "traj"])
def test_complex_shapes(S, oracle_mod, B, L, K, T, sc, bwd):
    c = gen.complex_inputs(B, L, K, seed=L + K)
    got = run_complex(S, c, T, sc, bwd)
    ref = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"])
    check_complex(got, ref)
    check_complex_ckpt(got, T)


def test_complex_backward_variants_agree(S):
    """Both backward calls sweep the same adjoint with the same transitions; the checkpointed one
    recomputes h_{t-1} from the checkpoints, so they agree to fp32 recurrence rounding."""
    c = gen.complex_inputs(2, 700, 130, seed=5)
    a = run_complex(S, c, 64, 3, "ckpt")
    b = run_complex(S, c, 64, 3, "traj")
    for k in ("du", "dr", "dphi", "dlambda", "domega"):
        assert rel_l2(a[k], b[k]) <= 1e-5, k


def test_complex_forward_checkpoints_only(S, oracle_mod):
    """With no trajectory buffer the forward writes only the checkpoints, and the checkpointed
    backward needs nothing else: the O(L/T) path."""
    c = gen.complex_inputs(2, 333, 64, seed=9)
    u = to_dev(c["u"], torch.complex64)
    g = to_dev(c["g"], torch.complex64)
    r, phi = to_dev(c["r"], torch.float32), to_dev(c["phi"], torch.float32)
    lam, om = to_dev(c["lam"], torch.float32), to_dev(c["omega"], torch.float32)
    h, ck = S.ssm_scan_complex_fwd(u, r, phi, lam, om, chunk=32, want_h=False, want_ckpt=True)
    assert h is None
    gr = S.ssm_scan_complex_bwd(u, r, phi, lam, om, ck, g, chunk=32)
    torch.cuda.synchronize()
    ref = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"])
    ends = [min(333, (i + 1) * 32) - 1 for i in range(ck.shape[1])]
    assert rel_l2(np64(ck), ref["h"][:, ends, :]) <= FWD_TOL_F32
    for k in ("du", "dr", "dphi", "dlambda", "domega"):
        assert rel_l2(np64(gr[k]), ref[k]) <= GRAD_TOL_F32, k


def test_complex_far_phases(S, oracle_mod):
    """Phases |omega phi| beyond the pi/2 reduction's range (~6400) take the library sine/cosine,
    warp-uniformly, inside the producers' packed transitions; the rest of the tile keeps the
    series.  Forward and backward against the oracle, with and without time segments."""
    c = gen.complex_inputs(2, 260, 130, seed=11)
    c["phi"][0, 40:52] = np.linspace(-7000.0, 9000.0, 12, dtype=np.float32)
    c["phi"][1, 200] = 12345.0
    ref = oracle_mod.complex_(c["u"], c["r"], c["phi"], c["lam"], c["omega"], c["g"])
    for sc in (0, 1):
        for bwd in ("ckpt", "traj"):
            check_complex(run_complex(S, c, 64, sc, bwd), ref)


# ------------------------------------------------------------------------------ full-size workloads

def _channel_sample(D, n=24):
    # first tile, a middle stretch, and the last channels (covers the ragged/last tile)
    idx = sorted(set(list(range(0, 8)) + list(range(D // 2, D // 2 + 8)) + list(range(D - 8, D))))
    return np.array(idx[:n])


@pytest.mark.parametrize("name", ["mamba130m_layer", "stiff_impulse", "mamba1p4b_layer"])
def test_full_size_real_sampled(S, oracle_mod, name):
    w = gen.WORKLOADS[name]
    inp = gen.workload_inputs(name)
    sel = _channel_sample(w.dim)
    mask = np.zeros(w.dim, dtype=np.float32)
    mask[sel] = 1.0
    masked = dict(inp)
    masked["dy"] = inp["dy"] * mask
    got = run_real(S, masked, w.io, w.chunk)
    # oracle on the sampled channels only (as its own contiguous problem)
    sub = {k: (v[..., sel] if k in ("x", "delta_raw", "dy") else v) for k, v in masked.items()}
    sub["A_log"], sub["Dskip"] = inp["A_log"][sel], inp["Dskip"][sel]
    ref = oracle_mod.real(sub["x"], sub["delta_raw"], sub["A_log"], sub["Bm"], sub["Cm"],
                          sub["Dskip"], sub["dy"], chunk=w.chunk, want_ckpt=True)
    pick = {"y": got["y"][..., sel], "ckpt": got["ckpt"][:, :, sel], "dx": got["dx"][..., sel],
            "ddelta_raw": got["ddelta_raw"][..., sel], "dA_log": got["dA_log"][sel],
            "dD": got["dD"][sel], "dB": got["dB"], "dC": got["dC"]}
    check_real(pick, ref, w.io)
    rest = np.ones(w.dim, dtype=bool)
    rest[sel] = False
    for k in ("dx", "ddelta_raw"):
        assert not np.any(got[k][..., rest]), k
    assert not np.any(got["dA_log"][rest]) and not np.any(got["dD"][rest])


@pytest.mark.parametrize("name", ["mamba130m_layer", "mamba1p4b_layer"])
def test_full_size_real_identities(S, name):
    """Unmasked full-size run: Euler homogeneity of y in x, Bm and Cm, on the GPU's own outputs."""
    w = gen.WORKLOADS[name]
    inp = gen.workload_inputs(name)
    got = run_real(S, inp, w.io, w.chunk)
    x, dy, Bm, Cm = (inp[k].astype(np.float64) for k in ("x", "dy", "Bm", "Cm"))
    loss = np.sum(dy * got["y"])
    skip = np.sum(dy * inp["Dskip"] * x)
    tol = 3e-2 if w.io == gen.BF16 else 1e-4
    assert abs(np.sum(x * got["dx"]) - loss) <= tol * abs(loss)
    assert abs(np.sum(Bm * got["dB"]) - (loss - skip)) <= tol * abs(loss - skip)
    assert abs(np.sum(Cm * got["dC"]) - (loss - skip)) <= tol * abs(loss - skip)
    assert abs(np.sum(inp["Dskip"] * got["dD"]) - skip) <= 1e-4 * abs(skip)


@pytest.mark.parametrize("bwd", ["ckpt", "traj"])
def test_full_size_complex_sampled(S, oracle_mod, bwd):
    w = gen.WORKLOADS["sparc_complex"]
    c = gen.workload_inputs("sparc_complex")
    sel = _channel_sample(w.modes)
    mask = np.zeros(w.modes, dtype=np.float32)
    mask[sel] = 1.0
    cm = dict(c)
    cm["g"] = (c["g"] * mask).astype(np.complex64)
    got = run_complex(S, cm, w.chunk, 0, bwd)
    check_complex_ckpt(got, w.chunk)
    ref = oracle_mod.complex_(c["u"][..., sel], c["r"], c["phi"], c["lam"][sel],
                              c["omega"][sel], cm["g"][..., sel])
    pick = {"h": got["h"][..., sel], "du": got["du"][..., sel], "dr": got["dr"],
            "dphi": got["dphi"], "dlambda": got["dlambda"][sel], "domega": got["domega"][sel]}
    check_complex(pick, ref)
    rest = np.ones(w.modes, dtype=bool)
    rest[sel] = False
    assert not np.any(got["du"][..., rest])
    # the forward is independent of g: every mode's h is checked on a second sample
    sel2 = np.arange(w.modes // 4, w.modes // 4 + 16)
    ref2 = oracle_mod.complex_(c["u"][..., sel2], c["r"], c["phi"], c["lam"][sel2], c["omega"][sel2])
    assert rel_l2(got["h"][..., sel2], ref2["h"]) <= FWD_TOL_F32
