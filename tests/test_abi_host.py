"""Host-side checks of the C ABI: the library builds for sm_100a, loads without a GPU, exports every
function declared in include/ssm_scan.h, answers size queries by their documented formulas and
rejects bad arguments with the documented status before touching the device.  No call here
reaches a CUDA runtime function (every case fails validation first)."""

import ctypes
import os
import re
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_scan.h")

pytestmark = pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists(
    os.path.join(ROOT, "selective_state_space_bwd_b200", "libssm_scan.so")),
    reason="needs nvcc or a prebuilt libssm_scan.so")


@pytest.fixture(scope="module")
def S():
    from selective_state_space_bwd_b200 import build, ssm_scan
    build.build()
    ssm_scan.lib()
    return ssm_scan


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(ssm_\w+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_symbol(S):
    names = _declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(S.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(S.EXPORTED)


def test_abi_version_and_status_strings(S):
    L = S.lib()
    assert L.ssm_scan_abi_version() == 5
    for code in range(8):
        assert L.ssm_status_string(code).decode().startswith(S.STATUS_NAMES[code])
    assert L.ssm_status_string(99) == b"unknown ssm_status"


@pytest.mark.parametrize("B,L,D,N,T", [(1, 256, 4, 4, 128), (8, 2048, 1536, 16, 128),
                                       (1, 128000, 1024, 16, 128), (3, 1000, 40, 8, 64),
                                       (2, 0, 16, 16, 32)])
def test_checkpoint_and_workspace_sizes(S, B, L, D, N, T):
    shp = S.real_shape(B, L, D, N, T, S.SSM_F32)
    nC = -(-L // T)
    assert S.checkpoint_bytes(shp) == B * nC * D * N * 4
    fw, bw = S.workspace_bytes(shp, False), S.workspace_bytes(shp, True)
    assert fw >= 256 and bw >= 256 and fw % 256 == 0 and bw % 256 == 0
    # the backward's dB/dC partial sums cover one launch's steps, capped at
    # max(checkpoint bytes, 128 MiB); its per-CTA scratch is capped at 192 MiB per launch; the
    # segment summaries take at most as much as the checkpoints
    cap = max(S.checkpoint_bytes(shp), 128 << 20)
    assert bw <= 2 * cap + (193 << 20)


def test_backward_workspace_is_o_of_l_over_t(S):
    """Growing L 4x at the stiff workload's width grows the backward workspace by no more than
    the checkpoints grow (the O(L/T) memory of the chunk-tiled backward)."""
    a = S.real_shape(1, 128000, 1024, 16, 128, S.SSM_F32)
    b = S.real_shape(1, 512000, 1024, 16, 128, S.SSM_F32)
    dw = S.workspace_bytes(b, True) - S.workspace_bytes(a, True)
    dc = S.checkpoint_bytes(b) - S.checkpoint_bytes(a)
    assert dw <= dc
    every_state = 512000 * 1024 * 16 * 4
    assert S.workspace_bytes(b, True) + S.checkpoint_bytes(b) < every_state / 10


def test_segment_knob_changes_only_workspace(S):
    a = S.real_shape(1, 4096, 64, 16, 128, S.SSM_F32, seg_chunks=1)
    b = S.real_shape(1, 4096, 64, 16, 128, S.SSM_F32, seg_chunks=32)
    assert S.checkpoint_bytes(a) == S.checkpoint_bytes(b)
    assert S.workspace_bytes(a, False) > S.workspace_bytes(b, False)


@pytest.mark.parametrize("field,value,code", [
    ("dstate", 12, 2), ("dstate", 32, 2), ("chunk", 100, 2), ("chunk", 512, 2), ("io", 3, 2),
    ("batch", -1, 1), ("seqlen", -5, 1), ("dim", 0, 1), ("reserved", 1, 1), ("seg_chunks", -1, 1),
    ("dim", 6, 3),  # 6 * 4 bytes is not a multiple of 16
])
def test_invalid_shapes_rejected(S, field, value, code):
    shp = S.real_shape(2, 64, 16, 16, 32, S.SSM_F32)
    setattr(shp, field, value)
    L = S.lib()
    assert L.ssm_scan_workspace_bytes(ctypes.byref(shp), 0) == 0
    assert L.ssm_scan_checkpoint_bytes(ctypes.byref(shp)) == 0
    fake = ctypes.c_void_p(0x10000)
    rc = L.ssm_scan_fwd(ctypes.byref(shp), *([fake] * 9), 1 << 20, None)
    assert rc == code


def test_bf16_row_alignment(S):
    L = S.lib()
    ok = S.real_shape(1, 8, 8, 16, 16, S.SSM_BF16)       # 8 * 2 = 16 bytes
    bad = S.real_shape(1, 8, 4, 16, 16, S.SSM_BF16)      # 4 * 2 = 8 bytes
    assert L.ssm_scan_workspace_bytes(ctypes.byref(ok), 1) > 0
    assert L.ssm_scan_workspace_bytes(ctypes.byref(bad), 1) == 0


def _fake_ptrs(n, base=0x100000):
    return [ctypes.c_void_p(base + 0x1000 * i) for i in range(n)]


def test_null_misaligned_and_small_workspace(S):
    L = S.lib()
    shp = S.real_shape(2, 64, 16, 16, 32, S.SSM_F32)
    need = S.workspace_bytes(shp, False)
    p = _fake_ptrs(9)
    q = list(p)
    q[0] = None
    assert L.ssm_scan_fwd(ctypes.byref(shp), *q, need, None) == 1
    q = list(p)
    q[3] = ctypes.c_void_p(0x100008)
    assert L.ssm_scan_fwd(ctypes.byref(shp), *q, need, None) == 3
    assert L.ssm_scan_fwd(ctypes.byref(shp), *p, need - 1, None) == 4
    pb = _fake_ptrs(15)
    needb = S.workspace_bytes(shp, True)
    assert L.ssm_scan_bwd(ctypes.byref(shp), *pb, needb - 256, None) == 4
    qb = list(pb)
    qb[7] = None  # dy
    assert L.ssm_scan_bwd(ctypes.byref(shp), *qb, needb, None) == 1


def test_option_validation(S):
    """The option-taking calls reject an unknown discretization, an unknown flag and a
    misaligned state pointer before anything is enqueued; NULL options equal the plain calls'
    validation."""
    L = S.lib()
    shp = S.real_shape(2, 64, 16, 16, 32, S.SSM_F32)
    need, needb = S.workspace_bytes(shp, False), S.workspace_bytes(shp, True)
    p, pb = _fake_ptrs(9), _fake_ptrs(15)
    bad_disc = S.SsmOptions(2, 0, None, None, None, None)
    bad_res = S.SsmOptions(S.SSM_ZOH, 7, None, None, None, None)     # bits beyond SSM_FUSED_SUMS
    bad_flag = S.SsmOptions(S.SSM_EULER, 2, None, None, None, None)
    mis_h0 = S.SsmOptions(S.SSM_EULER, 0, 0x100004, None, None, None)
    mis_dh0 = S.SsmOptions(S.SSM_ZOH, 0, None, None, None, 0x100008)
    for o in (bad_disc, bad_res, bad_flag):
        assert L.ssm_scan_fwd_ex(ctypes.byref(shp), ctypes.byref(o), *p, need, None) == 1
        assert L.ssm_scan_bwd_ex(ctypes.byref(shp), ctypes.byref(o), *pb, needb, None) == 1
    assert L.ssm_scan_fwd_ex(ctypes.byref(shp), ctypes.byref(mis_h0), *p, need, None) == 3
    assert L.ssm_scan_bwd_ex(ctypes.byref(shp), ctypes.byref(mis_dh0), *pb, needb, None) == 3
    # SSM_FUSED_SUMS is a valid flag: the call gets as far as the workspace check
    fused = S.SsmOptions(S.SSM_EULER, S.SSM_FUSED_SUMS, None, None, None, None)
    assert L.ssm_scan_bwd_ex(ctypes.byref(shp), ctypes.byref(fused), *pb, needb - 256, None) == 4
    # NULL options: same checks as the plain calls (here: workspace too small)
    assert L.ssm_scan_fwd_ex(ctypes.byref(shp), None, *p, need - 1, None) == 4
    assert L.ssm_scan_bwd_ex(ctypes.byref(shp), None, *pb, needb - 256, None) == 4


def test_rtrl_validation(S):
    L = S.lib()
    shp = S.complex_shape(2, 64, 128, 32)
    need = S.complex_rtrl_workspace_bytes(shp)
    assert need >= 256 + 2 * 128 * 8
    p = _fake_ptrs(11)
    assert L.ssm_scan_complex_rtrl(ctypes.byref(shp), *p, need - 1, None) == 4
    q = list(p)
    q[5] = None  # g
    assert L.ssm_scan_complex_rtrl(ctypes.byref(shp), *q, need, None) == 1
    q = list(p)
    q[8] = ctypes.c_void_p(0x100008)  # state misaligned
    assert L.ssm_scan_complex_rtrl(ctypes.byref(shp), *q, need, None) == 3
    odd = S.complex_shape(2, 64, 127, 32)
    assert L.ssm_scan_complex_rtrl(ctypes.byref(odd), *p, need, None) == 3


def test_pdssm_validation(S):
    L = S.lib()
    shp = S.pdssm_shape(2, 64, 8, 16, 8)
    assert S.pdssm_workspace_bytes(shp) == 256
    assert S.pdssm_workspace_bytes(S.pdssm_shape(2, 64, 8, 12, 8)) == 0      # N not in {4,8,16,32}
    assert S.pdssm_workspace_bytes(S.pdssm_shape(2, 64, 8, 16, 33)) == 0     # K > 32
    assert S.pdssm_workspace_bytes(S.pdssm_shape(1, 64, (1 << 21) + 1, 4, 2)) == 0  # H > 2^21
    assert S.pdssm_workspace_bytes(S.pdssm_shape(1, 64, 1 << 21, 4, 2)) == 256
    p = _fake_ptrs(8)
    assert L.ssm_pdssm_fwd(ctypes.byref(shp), *p, 255, None) == 4
    bad = S.pdssm_shape(2, 64, 8, 16, 0)
    assert L.ssm_pdssm_fwd(ctypes.byref(bad), *p, 256, None) == 2
    q = list(p)
    q[5] = None  # h
    assert L.ssm_pdssm_fwd(ctypes.byref(shp), *q, 256, None) == 1
    pb = _fake_ptrs(12)
    assert L.ssm_pdssm_bwd(ctypes.byref(shp), ctypes.c_float(0.0), *pb, 256, None) == 1   # tau
    qb = list(pb)
    qb[6] = None  # g
    assert L.ssm_pdssm_bwd(ctypes.byref(shp), ctypes.c_float(1.0), *qb, 256, None) == 1
    qb = list(pb)
    qb[10] = ctypes.c_void_p(0x100004)  # dh0 misaligned
    assert L.ssm_pdssm_bwd(ctypes.byref(shp), ctypes.c_float(1.0), *qb, 256, None) == 3


def test_complex_validation(S):
    L = S.lib()
    shp = S.complex_shape(2, 64, 16, 32)
    need_f = S.complex_workspace_bytes(shp, False)
    need_b = S.complex_workspace_bytes(shp, True)
    assert need_f >= 256 and need_b >= need_f
    odd = S.complex_shape(2, 64, 15, 32)
    assert S.complex_workspace_bytes(odd, True) == 0
    badT = S.complex_shape(2, 64, 16, 48)
    assert S.complex_workspace_bytes(badT, False) == 0
    p = _fake_ptrs(8)  # u, r, phi, lambda, omega, h, ckpt, ws
    assert L.ssm_scan_complex_fwd(ctypes.byref(shp), *p, need_f - 1, None) == 4
    q = list(p)
    q[1] = None
    assert L.ssm_scan_complex_fwd(ctypes.byref(shp), *q, need_f, None) == 1
    q = list(p)
    q[5] = q[6] = None  # neither the trajectory nor the checkpoints: nothing to write
    assert L.ssm_scan_complex_fwd(ctypes.byref(shp), *q, need_f, None) == 1
    q = list(p)
    q[5] = None  # checkpoints only is a valid forward
    q[6] = ctypes.c_void_p(0x100004)
    assert L.ssm_scan_complex_fwd(ctypes.byref(shp), *q, need_f, None) == 3
    pb = _fake_ptrs(13)  # checkpointed backward: u, r, phi, lambda, omega, ckpt, g, 5 outputs, ws
    pb[5] = ctypes.c_void_p(0x100004)
    assert L.ssm_scan_complex_bwd(ctypes.byref(shp), *pb, need_b, None) == 3
    pb = _fake_ptrs(13)
    pb[5] = None  # the checkpoints are required
    assert L.ssm_scan_complex_bwd(ctypes.byref(shp), *pb, need_b, None) == 1
    pb = _fake_ptrs(13)
    assert L.ssm_scan_complex_bwd(ctypes.byref(shp), *pb, need_b - 1, None) == 4
    pt = _fake_ptrs(12)  # trajectory backward: h, r, phi, lambda, omega, g, 5 outputs, ws
    pt[5] = ctypes.c_void_p(0x100004)
    assert L.ssm_scan_complex_bwd_traj(ctypes.byref(shp), *pt, need_b, None) == 3


def test_complex_checkpoint_bytes(S):
    # B * ceil(L / T) * K complex64 values
    assert S.complex_checkpoint_bytes(S.complex_shape(16, 4096, 2048, 128)) == 16 * 32 * 2048 * 8
    assert S.complex_checkpoint_bytes(S.complex_shape(3, 517, 130, 32)) == 3 * 17 * 130 * 8
    assert S.complex_checkpoint_bytes(S.complex_shape(2, 0, 64, 64)) == 0
    assert S.complex_checkpoint_bytes(S.complex_shape(2, 64, 15, 32)) == 0  # odd K: invalid
    # the backward workspace covers the chunk-trajectory scratch, which stays O(L / T): doubling
    # L at a fixed problem width never more than doubles it, and it is capped at 64 MiB or the
    # checkpoints, whichever is larger
    for B, K in ((16, 2048), (1, 64), (2, 256)):
        prev = None
        for L in (4096, 8192, 16384, 32768):
            shp = S.complex_shape(B, L, K, 128)
            ws = S.complex_workspace_bytes(shp, True)
            ck = S.complex_checkpoint_bytes(shp)
            traj_cap = max(64 << 20, ck)
            assert ws <= traj_cap + B * L * 8 * ((K + 63) // 64) + 8 * B * K * (L // 128) * 4 + (1 << 20)
            if prev is not None:
                assert ws <= 2 * prev + (1 << 20)
            prev = ws


def test_status_null_workspace(S):
    assert S.lib().ssm_scan_status(None, None) == 1


def test_kernel_launch_counts(S):
    one = S.real_shape(8, 2048, 1536, 16, 128, S.SSM_BF16)        # enough CTAs: no time split
    assert S.kernel_launches(one, False) == 1 and S.kernel_launches(one, True) == 3
    # with SSM_FUSED_SUMS its 384 CTAs are all resident: the scan kernel adds the dB/dC sums
    assert S.kernel_launches(one, True, fused_sums=True) == 2
    # few CTAs: concurrent segments + carry; the backward uses 250 segments of 4 chunks, 63 per
    # launch (2016 CTAs) so that each launch's dB/dC partial sums stay under their cap:
    # summary + carry + 4 x (main + reduce) + params = 11
    split = S.real_shape(1, 128000, 1024, 16, 128, S.SSM_F32)
    assert S.kernel_launches(split, False) == 3 and S.kernel_launches(split, True) == 11
    # 40 segments of 4 chunks x 64 CTAs, 20 per launch: 1280 CTAs per launch, more than the 592
    # resident ones, so the scratch is 592 slots that CTAs claim (58.2 MB, not 125.8 MB)
    multi = S.real_shape(2, 20000, 1024, 16, 128, S.SSM_F32)
    assert S.kernel_launches(multi, True) == 7
    assert S.kernel_launches(multi, True, fused_sums=True) == 7   # not resident: unchanged
    assert S.workspace_bytes(multi, True) - 592 * 98304 < 95_000_000
    # 512 CTAs fit one wave (4 CTAs per SM on 148 SMs = 592 slots): no time split, time in 4
    # sequential blocks under the partial cap
    wave = S.real_shape(4, 8192, 4096, 16, 128, S.SSM_BF16)
    assert S.kernel_launches(wave, False) == 1 and S.kernel_launches(wave, True) == 9
    assert S.kernel_launches(wave, True, fused_sums=True) == 5
    # 640 CTAs would leave a second wave of 48 on 592 slots: 16 concurrent segments of 4 chunks
    # instead, 3 per launch (summary + carry + 6 x (main + reduce) + params)
    part = S.real_shape(5, 8192, 4096, 16, 128, S.SSM_BF16)
    assert S.kernel_launches(part, True) == 15
    # wide enough to fill the SMs: no split; time in 4 sequential blocks under the partial cap
    blocks = S.real_shape(16, 2048, 4096, 16, 128, S.SSM_BF16)
    assert S.kernel_launches(blocks, False) == 1 and S.kernel_launches(blocks, True) == 9
    assert S.kernel_launches(S.real_shape(2, 0, 32, 16, 128), True) == 0
    assert S.kernel_launches(S.real_shape(2, 8, 32, 12, 128), True) == -1
    big = S.complex_shape(16, 4096, 2048, 128)
    # checkpointed backward: one main launch (512 CTAs, no time split) + the two reductions;
    # the trajectory backward: main + two reductions as well
    assert S.complex_kernel_launches(big, 1) == 3 and S.complex_kernel_launches(big, 2) == 3
    assert S.complex_kernel_launches(big, 0) == 1 and S.complex_kernel_launches(big, 3) == -1
    # PD-SSM: one scan kernel per call (argmax / score gradient fused) at the bench size; time
    # segments below 128 CTAs add summary + carry; K * (128 / N) > 256 adds the separate kernel
    pd = S.pdssm_shape(8, 5120, 256, 16, 8)
    assert S.pdssm_kernel_launches(pd, False) == 1 and S.pdssm_kernel_launches(pd, True) == 1
    assert S.pdssm_workspace_bytes(pd) == 256
    few = S.pdssm_shape(1, 1000, 8, 16, 8)
    assert S.pdssm_kernel_launches(few, False) == 3 and S.pdssm_kernel_launches(few, True) == 3
    wide = S.pdssm_shape(2, 64, 8, 4, 9)
    assert S.pdssm_kernel_launches(wide, False) == 2 and S.pdssm_kernel_launches(wide, True) == 2
    assert S.pdssm_kernel_launches(S.pdssm_shape(2, 0, 8, 16, 8), False) == 0
    assert S.pdssm_kernel_launches(S.pdssm_shape(2, 8, 8, 12, 8), False) == -1


def test_dtproj_validation(S):
    import ctypes
    L = S.lib()
    ok = S.dtproj_shape(1000, 1536, 48)
    # status word (256 bytes), then one split of 1024 rows x (R + 1) columns x D
    assert S.dtproj_workspace_bytes(ok) == 256 + 1536 * 49 * 4
    assert S.dtproj_workspace_bytes(ok, backward=False) == 256
    assert S.dtproj_workspace_bytes(S.dtproj_shape(3000, 64, 128)) == 256 + 3 * 64 * 129 * 4
    assert S.dtproj_workspace_bytes(S.dtproj_shape(10, 1536, 40)) == 0   # R not a multiple of 16
    assert S.dtproj_workspace_bytes(S.dtproj_shape(10, 1532, 48)) == 0   # D not a multiple of 8
    assert S.dtproj_workspace_bytes(S.dtproj_shape(10, 64, 272)) == 0    # R > 256
    assert S.dtproj_workspace_bytes(S.dtproj_shape(10, 64, 16, S.SSM_F32)) == 0
    assert S.dtproj_workspace_bytes(S.dtproj_shape(0, 64, 16)) == 256
    p16 = [ctypes.c_void_p(4096)] * 5
    assert L.ssm_dtproj_fwd(ctypes.byref(S.dtproj_shape(10, 64, 16, S.SSM_F32)), *p16, 256, None) == 2
    assert L.ssm_dtproj_fwd(ctypes.byref(S.dtproj_shape(10, 64, 40)), *p16, 256, None) == 2
    assert L.ssm_dtproj_fwd(ctypes.byref(ok), None, *p16[:4], 256, None) == 1       # u missing
    odd = [ctypes.c_void_p(4096), ctypes.c_void_p(4104), ctypes.c_void_p(4096), None, ctypes.c_void_p(4096)]
    assert L.ssm_dtproj_fwd(ctypes.byref(ok), *odd, 256, None) == 3                 # w misaligned
    assert L.ssm_dtproj_fwd(ctypes.byref(ok), *p16, 255, None) == 4                 # workspace
    pb = [ctypes.c_void_p(4096)] * 7
    assert L.ssm_dtproj_bwd(ctypes.byref(ok), *pb, 255, None) == 4                  # workspace


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_cpp(tmp_path):
    """include/ssm_scan.h is a plain C header (usable from C and C++ callers alike)."""
    import subprocess
    src = tmp_path / "use_header.c"
    src.write_text('#include "ssm_scan.h"\n'
                   "int main(void) {\n"
                   "    ssm_shape s = {1, 16, 8, 4, 128, SSM_F32, 0, 0};\n"
                   "    ssm_dtshape d = {0, 8, 16, SSM_BF16};\n"
                   "    return (int)(ssm_scan_checkpoint_bytes(&s) * 0 + ssm_dtproj_workspace_bytes(&d, 0) * 0);\n"
                   "}\n")
    inc = os.path.join(ROOT, "include")
    for cmd in (["gcc", "-std=c11", "-Wall", "-Werror", "-I", inc, "-c", str(src), "-o", str(tmp_path / "a.o")],
                ["g++", "-std=c++17", "-Wall", "-Werror", "-I", inc, "-x", "c++", "-c", str(src),
                 "-o", str(tmp_path / "b.o")]):
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
