"""ctypes binding of libssm_scan.so (include/ssm_scan.h), over torch device tensors.

Argument marshalling only: every step of the scan runs in the library's CUDA kernels.  If the
library is missing, or the tensors are not on a CUDA device, the calls raise — there is no CPU
fallback.  Names mirror the C ABI: ``ssm_scan_fwd``, ``ssm_scan_bwd``, ``ssm_scan_complex_fwd``,
``ssm_scan_complex_bwd``, ``ssm_scan_complex_bwd_traj``, ``ssm_scan_status``; the workspace / checkpoint size queries are exposed
as ``workspace_bytes`` and friends.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_scan.so")

SSM_OK = 0
SSM_F32, SSM_BF16 = 0, 1
STATUS_NAMES = {0: "SSM_OK", 1: "SSM_ERR_INVALID_ARG", 2: "SSM_ERR_UNSUPPORTED",
                3: "SSM_ERR_MISALIGNED", 4: "SSM_ERR_WORKSPACE_TOO_SMALL", 5: "SSM_ERR_CUDA",
                6: "SSM_ERR_TIMEOUT", 7: "SSM_ERR_NONFINITE"}


class SsmShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("chunk", ctypes.c_int32), ("io", ctypes.c_int32),
                ("seg_chunks", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class SsmCShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("modes", ctypes.c_int64),
                ("chunk", ctypes.c_int32), ("seg_chunks", ctypes.c_int32)]


SSM_EULER, SSM_ZOH = 0, 1
SSM_FUSED_SUMS = 1  # ssm_scan_options.flags: dB/dC sums inside the backward's scan kernel


class SsmOptions(ctypes.Structure):
    _fields_ = [("discretization", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("h0", ctypes.c_void_p), ("hL", ctypes.c_void_p), ("dhL", ctypes.c_void_p),
                ("dh0", ctypes.c_void_p)]


class SsmPdShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("heads", ctypes.c_int64),
                ("nstate", ctypes.c_int32), ("ndict", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("reserved2", ctypes.c_int32)]


class SsmDtShape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("dim", ctypes.c_int64), ("rank", ctypes.c_int32),
                ("io", ctypes.c_int32)]


class SsmError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")


_lock = threading.Lock()
_lib = None

EXPORTED = ["ssm_scan_abi_version", "ssm_scan_checkpoint_bytes", "ssm_scan_workspace_bytes",
            "ssm_scan_fwd", "ssm_scan_bwd", "ssm_scan_complex_workspace_bytes",
            "ssm_scan_complex_fwd", "ssm_scan_complex_bwd", "ssm_scan_complex_bwd_traj",
            "ssm_scan_complex_checkpoint_bytes", "ssm_scan_kernel_launches",
            "ssm_scan_complex_kernel_launches", "ssm_scan_status", "ssm_status_string",
            "ssm_scan_fwd_noalloc", "ssm_scan_fwd_ex", "ssm_scan_bwd_ex",
            "ssm_scan_complex_rtrl_workspace_bytes", "ssm_scan_complex_rtrl",
            "ssm_pdssm_workspace_bytes", "ssm_pdssm_fwd", "ssm_pdssm_bwd",
            "ssm_pdssm_kernel_launches", "ssm_dtproj_workspace_bytes", "ssm_dtproj_fwd",
            "ssm_dtproj_bwd"]


def lib():
    """Open libssm_scan.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m selective_state_space_bwd_b200.build` (no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            P, Z, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            SP, CP = ctypes.POINTER(SsmShape), ctypes.POINTER(SsmCShape)
            L.ssm_scan_abi_version.argtypes, L.ssm_scan_abi_version.restype = [], I
            L.ssm_scan_checkpoint_bytes.argtypes, L.ssm_scan_checkpoint_bytes.restype = [SP], Z
            L.ssm_scan_workspace_bytes.argtypes, L.ssm_scan_workspace_bytes.restype = [SP, I], Z
            L.ssm_scan_fwd.argtypes = [SP] + [P] * 9 + [Z, P]
            L.ssm_scan_fwd.restype = I
            L.ssm_scan_bwd.argtypes = [SP] + [P] * 15 + [Z, P]
            L.ssm_scan_bwd.restype = I
            L.ssm_scan_complex_workspace_bytes.argtypes = [CP, I]
            L.ssm_scan_complex_workspace_bytes.restype = Z
            L.ssm_scan_complex_checkpoint_bytes.argtypes = [CP]
            L.ssm_scan_complex_checkpoint_bytes.restype = Z
            L.ssm_scan_complex_fwd.argtypes = [CP] + [P] * 8 + [Z, P]
            L.ssm_scan_complex_fwd.restype = I
            L.ssm_scan_complex_bwd.argtypes = [CP] + [P] * 13 + [Z, P]
            L.ssm_scan_complex_bwd.restype = I
            L.ssm_scan_complex_bwd_traj.argtypes = [CP] + [P] * 12 + [Z, P]
            L.ssm_scan_complex_bwd_traj.restype = I
            L.ssm_scan_kernel_launches.argtypes = [SP, I]
            L.ssm_scan_kernel_launches.restype = I
            L.ssm_scan_complex_kernel_launches.argtypes = [CP, I]
            L.ssm_scan_complex_kernel_launches.restype = I
            L.ssm_scan_status.argtypes, L.ssm_scan_status.restype = [P, P], I
            L.ssm_status_string.argtypes, L.ssm_status_string.restype = [I], ctypes.c_char_p
            L.ssm_scan_fwd_noalloc.argtypes = [SP] + [P] * 8 + [P]
            L.ssm_scan_fwd_noalloc.restype = I
            L.ssm_scan_complex_rtrl_workspace_bytes.argtypes = [CP]
            L.ssm_scan_complex_rtrl_workspace_bytes.restype = Z
            L.ssm_scan_complex_rtrl.argtypes = [CP] + [P] * 11 + [Z, P]
            L.ssm_scan_complex_rtrl.restype = I
            PP = ctypes.POINTER(SsmPdShape)
            L.ssm_pdssm_workspace_bytes.argtypes, L.ssm_pdssm_workspace_bytes.restype = [PP], Z
            L.ssm_pdssm_fwd.argtypes = [PP] + [P] * 8 + [Z, P]
            L.ssm_pdssm_fwd.restype = I
            L.ssm_pdssm_bwd.argtypes = [PP, ctypes.c_float] + [P] * 12 + [Z, P]
            L.ssm_pdssm_bwd.restype = I
            L.ssm_pdssm_kernel_launches.argtypes, L.ssm_pdssm_kernel_launches.restype = [PP, I], I
            DP = ctypes.POINTER(SsmDtShape)
            L.ssm_dtproj_workspace_bytes.argtypes, L.ssm_dtproj_workspace_bytes.restype = [DP, I], Z
            L.ssm_dtproj_fwd.argtypes, L.ssm_dtproj_fwd.restype = [DP] + [P] * 5 + [Z, P], I
            L.ssm_dtproj_bwd.argtypes = [DP] + [P] * 7 + [Z, P]
            L.ssm_dtproj_bwd.restype = I
            OP = ctypes.POINTER(SsmOptions)
            L.ssm_scan_fwd_ex.argtypes = [SP, OP] + [P] * 9 + [Z, P]
            L.ssm_scan_fwd_ex.restype = I
            L.ssm_scan_bwd_ex.argtypes = [SP, OP] + [P] * 15 + [Z, P]
            L.ssm_scan_bwd_ex.restype = I
            _lib = L
    return _lib


def _check(code, what):
    if code != SSM_OK:
        raise SsmError(code, what)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("ssm_scan: every tensor must live on a CUDA device")


def real_shape(batch, seqlen, dim, dstate, chunk=128, io=SSM_F32, seg_chunks=0):
    return SsmShape(int(batch), int(seqlen), int(dim), int(dstate), int(chunk), int(io),
                    int(seg_chunks), 0)


def complex_shape(batch, seqlen, modes, chunk=128, seg_chunks=0):
    return SsmCShape(int(batch), int(seqlen), int(modes), int(chunk), int(seg_chunks))


def checkpoint_bytes(shape: SsmShape) -> int:
    return int(lib().ssm_scan_checkpoint_bytes(ctypes.byref(shape)))


def workspace_bytes(shape: SsmShape, backward: bool) -> int:
    return int(lib().ssm_scan_workspace_bytes(ctypes.byref(shape), int(bool(backward))))


def complex_workspace_bytes(shape: SsmCShape, backward: bool) -> int:
    return int(lib().ssm_scan_complex_workspace_bytes(ctypes.byref(shape), int(bool(backward))))


def kernel_launches(shape: SsmShape, backward: bool, fused_sums: bool = False) -> int:
    mode = (2 if fused_sums else 1) if backward else 0
    return int(lib().ssm_scan_kernel_launches(ctypes.byref(shape), mode))


def complex_checkpoint_bytes(shape: SsmCShape) -> int:
    return int(lib().ssm_scan_complex_checkpoint_bytes(ctypes.byref(shape)))


def complex_kernel_launches(shape: SsmCShape, backward) -> int:
    """backward: 0 / False the forward, 1 / True ssm_scan_complex_bwd (from checkpoints),
    2 ssm_scan_complex_bwd_traj (from the stored trajectory)."""
    return int(lib().ssm_scan_complex_kernel_launches(ctypes.byref(shape), int(backward)))


def _io_of(t):
    if t.dtype == torch.float32:
        return SSM_F32
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    raise ValueError(f"unsupported io dtype {t.dtype}")


def _workspace(nbytes, device, ws):
    if ws is not None:
        return ws
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def ssm_scan_fwd(x, delta_raw, A_log, Bm, Cm, Dskip, chunk=128, seg_chunks=0, y=None, ckpt=None,
                 ws=None, stream=None):
    """Forward scan.  x, delta_raw [B,L,D] and Bm, Cm [B,L,N] share one io dtype (fp32 / bf16);
    A_log [D,N], Dskip [D] fp32.  Returns (y [B,L,D], ckpt [B,ceil(L/T),D,N] fp32)."""
    _need_cuda(x, delta_raw, A_log, Bm, Cm, Dskip)
    B, L, D = x.shape
    N = A_log.shape[1]
    shape = real_shape(B, L, D, N, chunk, _io_of(x), seg_chunks)
    if y is None:
        y = torch.empty_like(x)
    nC = -(-L // chunk)
    if ckpt is None:
        ckpt = torch.empty((B, nC, D, N), dtype=torch.float32, device=x.device)
    ws = _workspace(workspace_bytes(shape, False), x.device, ws)
    code = lib().ssm_scan_fwd(ctypes.byref(shape), _p(x), _p(delta_raw), _p(A_log), _p(Bm), _p(Cm),
                              _p(Dskip), _p(y), _p(ckpt), _p(ws), ws.numel() * ws.element_size(),
                              _stream(stream))
    _check(code, "ssm_scan_fwd")
    return y, ckpt


def ssm_scan_fwd_noalloc(x, delta_raw, A_log, Bm, Cm, Dskip, y, ckpt, chunk=128, seg_chunks=0,
                         stream=None):
    """Forward scan without a workspace, for callers that cannot allocate device memory: the
    scratch is the library's built-in 8 MiB device array (shared by every call on a device, so
    overlapping calls race).  The caller passes preallocated ``y`` and ``ckpt``; this function
    allocates nothing.  Raises SsmError(SSM_ERR_WORKSPACE_TOO_SMALL) when the problem needs more
    scratch than the array holds."""
    _need_cuda(x, delta_raw, A_log, Bm, Cm, Dskip, y, ckpt)
    B, L, D = x.shape
    N = A_log.shape[1]
    shape = real_shape(B, L, D, N, chunk, _io_of(x), seg_chunks)
    code = lib().ssm_scan_fwd_noalloc(ctypes.byref(shape), _p(x), _p(delta_raw), _p(A_log), _p(Bm),
                                      _p(Cm), _p(Dskip), _p(y), _p(ckpt), _stream(stream))
    _check(code, "ssm_scan_fwd_noalloc")
    return y, ckpt


def ssm_scan_bwd(x, delta_raw, A_log, Bm, Cm, Dskip, ckpt, dy, chunk=128, seg_chunks=0, out=None,
                 ws=None, stream=None):
    """Backward.  Returns dict dx, ddelta_raw [B,L,D], dA_log [D,N], dB, dC [B,L,N], dD [D]."""
    _need_cuda(x, delta_raw, A_log, Bm, Cm, Dskip, ckpt, dy)
    B, L, D = x.shape
    N = A_log.shape[1]
    shape = real_shape(B, L, D, N, chunk, _io_of(x), seg_chunks)
    if out is None:
        out = dict(dx=torch.empty_like(x), ddelta_raw=torch.empty_like(x),
                   dA_log=torch.empty_like(A_log), dB=torch.empty_like(Bm), dC=torch.empty_like(Cm),
                   dD=torch.empty_like(Dskip))
    ws = _workspace(workspace_bytes(shape, True), x.device, ws)
    code = lib().ssm_scan_bwd(ctypes.byref(shape), _p(x), _p(delta_raw), _p(A_log), _p(Bm), _p(Cm),
                              _p(Dskip), _p(ckpt), _p(dy), _p(out["dx"]), _p(out["ddelta_raw"]),
                              _p(out["dA_log"]), _p(out["dB"]), _p(out["dC"]), _p(out["dD"]),
                              _p(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_scan_bwd")
    return out


def _options(zoh, h0=None, hL=None, dhL=None, dh0=None, fused_sums=False):
    for t in (h0, hL, dhL, dh0):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError("h0, hL, dhL, dh0 must be contiguous float32 [B, D, N]")
    return SsmOptions(SSM_ZOH if zoh else SSM_EULER, SSM_FUSED_SUMS if fused_sums else 0,
                      None if h0 is None else h0.data_ptr(),
                      None if hL is None else hL.data_ptr(), None if dhL is None else dhL.data_ptr(),
                      None if dh0 is None else dh0.data_ptr())


def ssm_scan_fwd_ex(x, delta_raw, A_log, Bm, Cm, Dskip, zoh=False, h0=None, chunk=128,
                    seg_chunks=0, y=None, ckpt=None, hL=None, ws=None, stream=None):
    """Forward scan with options: ``zoh`` selects the zero-order-hold input term, ``h0`` [B,D,N]
    fp32 is the initial state (None: zero).  Returns (y, ckpt, hL) with hL [B,D,N] the final
    state.  The backward must get the same ``zoh`` and ``h0``."""
    _need_cuda(x, delta_raw, A_log, Bm, Cm, Dskip, h0)
    B, L, D = x.shape
    N = A_log.shape[1]
    shape = real_shape(B, L, D, N, chunk, _io_of(x), seg_chunks)
    if y is None:
        y = torch.empty_like(x)
    if ckpt is None:
        ckpt = torch.empty((B, -(-L // chunk), D, N), dtype=torch.float32, device=x.device)
    if hL is None:
        hL = torch.empty((B, D, N), dtype=torch.float32, device=x.device)
    opts = _options(zoh, h0=h0, hL=hL)
    ws = _workspace(workspace_bytes(shape, False), x.device, ws)
    code = lib().ssm_scan_fwd_ex(ctypes.byref(shape), ctypes.byref(opts), _p(x), _p(delta_raw),
                                 _p(A_log), _p(Bm), _p(Cm), _p(Dskip), _p(y), _p(ckpt), _p(ws),
                                 ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_scan_fwd_ex")
    return y, ckpt, hL


def ssm_scan_bwd_ex(x, delta_raw, A_log, Bm, Cm, Dskip, ckpt, dy, zoh=False, h0=None, dhL=None,
                    chunk=128, seg_chunks=0, out=None, ws=None, stream=None, fused_sums=False):
    """Backward with options: the gradient of sum(dy y) + sum(dhL hL).  Returns the dict of
    ssm_scan_bwd plus dh0 [B,D,N] (the gradient with respect to h0).  ``fused_sums`` sets
    SSM_FUSED_SUMS (dB/dC sums inside the scan kernel where its CTAs can all be resident)."""
    _need_cuda(x, delta_raw, A_log, Bm, Cm, Dskip, ckpt, dy, h0, dhL)
    B, L, D = x.shape
    N = A_log.shape[1]
    shape = real_shape(B, L, D, N, chunk, _io_of(x), seg_chunks)
    if out is None:
        out = dict(dx=torch.empty_like(x), ddelta_raw=torch.empty_like(x),
                   dA_log=torch.empty_like(A_log), dB=torch.empty_like(Bm), dC=torch.empty_like(Cm),
                   dD=torch.empty_like(Dskip))
    if out.get("dh0") is None:
        out["dh0"] = torch.empty((B, D, N), dtype=torch.float32, device=x.device)
    opts = _options(zoh, h0=h0, dhL=dhL, dh0=out["dh0"], fused_sums=fused_sums)
    ws = _workspace(workspace_bytes(shape, True), x.device, ws)
    code = lib().ssm_scan_bwd_ex(ctypes.byref(shape), ctypes.byref(opts), _p(x), _p(delta_raw),
                                 _p(A_log), _p(Bm), _p(Cm), _p(Dskip), _p(ckpt), _p(dy),
                                 _p(out["dx"]), _p(out["ddelta_raw"]), _p(out["dA_log"]),
                                 _p(out["dB"]), _p(out["dC"]), _p(out["dD"]), _p(ws),
                                 ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_scan_bwd_ex")
    return out


def ssm_scan_complex_fwd(u, r, phi, lam, omega, chunk=128, seg_chunks=0, h=None, ckpt=None,
                         want_h=True, want_ckpt=False, ws=None, stream=None):
    """Complex forward.  u [B,L,K] complex64; r, phi [B,L]; lam, omega [K].  Returns h (the
    trajectory, or None when ``want_h`` is false and no ``h`` is given), or (h, ckpt) when
    ``want_ckpt`` is true or a ``ckpt`` [B, ceil(L/chunk), K] complex64 buffer is given."""
    _need_cuda(u, r, phi, lam, omega)
    if u.dtype != torch.complex64:
        raise ValueError("u must be complex64")
    B, L, K = u.shape
    shape = complex_shape(B, L, K, chunk, seg_chunks)
    if h is None and want_h:
        h = torch.empty_like(u)
    ret_ck = want_ckpt or ckpt is not None
    if ckpt is None and want_ckpt:
        ckpt = torch.empty((B, -(-L // chunk), K), dtype=torch.complex64, device=u.device)
    ws = _workspace(complex_workspace_bytes(shape, False), u.device, ws)
    code = lib().ssm_scan_complex_fwd(ctypes.byref(shape), _p(u), _p(r), _p(phi), _p(lam),
                                      _p(omega), _p(h), _p(ckpt), _p(ws),
                                      ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_scan_complex_fwd")
    return (h, ckpt) if ret_ck else h


def _complex_grads(g, r, phi, lam, omega, out):
    if out is None:
        out = dict(du=torch.empty_like(g), dr=torch.empty_like(r), dphi=torch.empty_like(phi),
                   dlambda=torch.empty_like(lam), domega=torch.empty_like(omega))
    return out


def ssm_scan_complex_bwd(u, r, phi, lam, omega, ckpt, g, chunk=128, seg_chunks=0, out=None,
                         ws=None, stream=None):
    """Complex backward of Re sum conj(g) h from the forward's checkpoints (each chunk's
    trajectory recomputed from its entering checkpoint).  Returns dict du, dr, dphi, dlambda,
    domega."""
    _need_cuda(u, r, phi, lam, omega, ckpt, g)
    B, L, K = u.shape
    shape = complex_shape(B, L, K, chunk, seg_chunks)
    out = _complex_grads(g, r, phi, lam, omega, out)
    ws = _workspace(complex_workspace_bytes(shape, True), u.device, ws)
    code = lib().ssm_scan_complex_bwd(ctypes.byref(shape), _p(u), _p(r), _p(phi), _p(lam),
                                      _p(omega), _p(ckpt), _p(g), _p(out["du"]), _p(out["dr"]),
                                      _p(out["dphi"]), _p(out["dlambda"]), _p(out["domega"]),
                                      _p(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_scan_complex_bwd")
    return out


def ssm_scan_complex_bwd_traj(h, r, phi, lam, omega, g, chunk=128, seg_chunks=0, out=None,
                              ws=None, stream=None):
    """Complex backward of Re sum conj(g) h reading the stored trajectory h.  Returns dict du,
    dr, dphi, dlambda, domega."""
    _need_cuda(h, r, phi, lam, omega, g)
    B, L, K = h.shape
    shape = complex_shape(B, L, K, chunk, seg_chunks)
    out = _complex_grads(g, r, phi, lam, omega, out)
    ws = _workspace(complex_workspace_bytes(shape, True), h.device, ws)
    code = lib().ssm_scan_complex_bwd_traj(ctypes.byref(shape), _p(h), _p(r), _p(phi), _p(lam),
                                           _p(omega), _p(g), _p(out["du"]), _p(out["dr"]),
                                           _p(out["dphi"]), _p(out["dlambda"]),
                                           _p(out["domega"]), _p(ws),
                                           ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_scan_complex_bwd_traj")
    return out


def ssm_scan_status(ws, stream=None) -> int:
    """Synchronise the stream and return the device status word a call left in ``ws``."""
    return int(lib().ssm_scan_status(_p(ws), _stream(stream)))


def complex_rtrl_workspace_bytes(shape: SsmCShape) -> int:
    return int(lib().ssm_scan_complex_rtrl_workspace_bytes(ctypes.byref(shape)))


def ssm_scan_complex_rtrl(u, r, phi, lam, omega, g, state=None, want_h=False, chunk=128,
                          h=None, out=None, ws=None, stream=None):
    """Complex forward with exact structured RTRL: returns dict dlambda, domega [K] (the gradient
    of Re sum conj(g) h accumulated online), and h [B,L,K] if ``want_h`` or ``h`` is given.
    ``state`` [B,3,K] complex64 (h, dh/dlambda, dh/domega) is read before the first step and
    updated in place after the last (None: start from zero)."""
    _need_cuda(u, r, phi, lam, omega, g, state, h)
    if u.dtype != torch.complex64 or g.dtype != torch.complex64:
        raise ValueError("u and g must be complex64")
    B, L, K = u.shape
    shape = complex_shape(B, L, K, chunk, 0)
    if h is None and want_h:
        h = torch.empty_like(u)
    if state is not None and (state.dtype != torch.complex64 or tuple(state.shape) != (B, 3, K)
                              or not state.is_contiguous()):
        raise ValueError("state must be a contiguous complex64 [B, 3, K] tensor")
    if out is None:
        out = dict(dlambda=torch.empty_like(lam), domega=torch.empty_like(omega))
    ws = _workspace(complex_rtrl_workspace_bytes(shape), u.device, ws)
    code = lib().ssm_scan_complex_rtrl(ctypes.byref(shape), _p(u), _p(r), _p(phi), _p(lam),
                                       _p(omega), _p(g), _p(h), _p(state), _p(out["dlambda"]),
                                       _p(out["domega"]), _p(ws), ws.numel() * ws.element_size(),
                                       _stream(stream))
    _check(code, "ssm_scan_complex_rtrl")
    if h is not None:
        out["h"] = h
    return out


def pdssm_shape(batch, seqlen, heads, nstate, ndict):
    return SsmPdShape(int(batch), int(seqlen), int(heads), int(nstate), int(ndict), 0, 0)


def pdssm_workspace_bytes(shape: SsmPdShape) -> int:
    return int(lib().ssm_pdssm_workspace_bytes(ctypes.byref(shape)))


def pdssm_kernel_launches(shape: SsmPdShape, backward: bool) -> int:
    return int(lib().ssm_pdssm_kernel_launches(ctypes.byref(shape), int(bool(backward))))


def ssm_pdssm_fwd(scores, dictionary, d, bt, h0=None, h=None, sel=None, ws=None, stream=None):
    """Flash PD-SSM forward: scores [B,L,H,K], dictionary [K,N] int32, d, bt [B,L,H,N] fp32,
    h0 [B,H,N] (None: zero).  Returns (h [B,L,H,N], sel [B,L,H] int32)."""
    _need_cuda(scores, dictionary, d, bt, h0)
    B, L, H, K = scores.shape
    N = d.shape[-1]
    shape = pdssm_shape(B, L, H, N, K)
    if h is None:
        h = torch.empty_like(d)
    if sel is None:
        sel = torch.empty((B, L, H), dtype=torch.int32, device=d.device)
    ws = _workspace(pdssm_workspace_bytes(shape), d.device, ws)
    code = lib().ssm_pdssm_fwd(ctypes.byref(shape), _p(scores), _p(dictionary), _p(d), _p(bt),
                               _p(h0), _p(h), _p(sel), _p(ws), ws.numel() * ws.element_size(),
                               _stream(stream))
    _check(code, "ssm_pdssm_fwd")
    return h, sel


def ssm_pdssm_bwd(scores, dictionary, d, h, sel, g, tau=1.0, h0=None, out=None, ws=None,
                  stream=None):
    """Flash PD-SSM backward of sum <g, h> (straight-through score gradient at temperature tau).
    Returns dict dd, dbt [B,L,H,N], dscores [B,L,H,K], dh0 [B,H,N]."""
    _need_cuda(scores, dictionary, d, h, sel, g, h0)
    B, L, H, K = scores.shape
    N = d.shape[-1]
    shape = pdssm_shape(B, L, H, N, K)
    if out is None:
        out = dict(dd=torch.empty_like(d), dbt=torch.empty_like(d),
                   dscores=torch.empty_like(scores),
                   dh0=torch.empty((B, H, N), dtype=torch.float32, device=d.device))
    ws = _workspace(pdssm_workspace_bytes(shape), d.device, ws)
    code = lib().ssm_pdssm_bwd(ctypes.byref(shape), float(tau), _p(scores), _p(dictionary), _p(d),
                               _p(h0), _p(h), _p(sel), _p(g), _p(out["dd"]), _p(out["dbt"]),
                               _p(out["dscores"]), _p(out.get("dh0")), _p(ws),
                               ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_pdssm_bwd")
    return out


def dtproj_shape(rows, dim, rank, io=SSM_BF16):
    return SsmDtShape(int(rows), int(dim), int(rank), int(io))


def dtproj_workspace_bytes(shape: SsmDtShape, backward: bool = True) -> int:
    return int(lib().ssm_dtproj_workspace_bytes(ctypes.byref(shape), 1 if backward else 0))


def ssm_dtproj_fwd(u, w, bias=None, delta_raw=None, ws=None, stream=None):
    """Step-size projection delta_raw = u w^T + bias.  u [..., R] and w [D, R] bf16, bias [D] fp32
    (or None).  Returns delta_raw [..., D] bf16.  ``ws`` (optional) holds the status word that
    ssm_scan_status reads."""
    _need_cuda(u, w, bias)
    R = u.shape[-1]
    D = w.shape[0]
    M = u.numel() // R if R else 0
    shape = dtproj_shape(M, D, R, _io_of(u))
    if delta_raw is None:
        delta_raw = torch.empty((*u.shape[:-1], D), dtype=u.dtype, device=u.device)
    ws = _workspace(dtproj_workspace_bytes(shape, False), u.device, ws)
    code = lib().ssm_dtproj_fwd(ctypes.byref(shape), _p(u), _p(w), _p(bias), _p(delta_raw), _p(ws),
                                ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_dtproj_fwd")
    return delta_raw


def ssm_dtproj_bwd(u, w, g, want_dbias=True, out=None, ws=None, stream=None):
    """Backward of the projection for g = dL/d delta_raw [..., D] bf16.  Returns dict du [..., R]
    bf16, dw [D, R] fp32, dbias [D] fp32 (None if not wanted)."""
    _need_cuda(u, w, g)
    R = u.shape[-1]
    D = w.shape[0]
    M = u.numel() // R if R else 0
    shape = dtproj_shape(M, D, R, _io_of(u))
    if out is None:
        out = dict(du=torch.empty_like(u), dw=torch.empty((D, R), dtype=torch.float32, device=u.device),
                   dbias=torch.empty(D, dtype=torch.float32, device=u.device) if want_dbias else None)
    ws = _workspace(dtproj_workspace_bytes(shape, True), u.device, ws)
    code = lib().ssm_dtproj_bwd(ctypes.byref(shape), _p(u), _p(w), _p(g), _p(out["du"]),
                                _p(out["dw"]), _p(out.get("dbias")), _p(ws),
                                ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "ssm_dtproj_bwd")
    return out

