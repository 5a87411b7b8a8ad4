"""Float64 CPU oracle for the selective scan (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs may
import this package.  The product path (``selective_state_space_bwd_b200``) never does, and this
package imports nothing from it: the two share no code.  The arithmetic lives in
``ssm_oracle.c`` (plain C99, float64, OpenMP over independent channels), built here with gcc.

Functions return float64 numpy arrays.  Inputs of any float dtype are upcast exactly to float64.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into libssm_oracle.so (gcc -O2 -fopenmp, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-std=c99", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.ssm_oracle_real.argtypes = [I64, I64, I64, I64, I64] + [P] * 7 + [I64, I64, ctypes.c_int] + [P] * 8
            lib.ssm_oracle_real.restype = ctypes.c_int
            lib.ssm_oracle_real_ex.argtypes = ([I64, I64, I64, I64, I64] + [P] * 7 +
                                               [I64, I64, ctypes.c_int, ctypes.c_int] + [P] * 12)
            lib.ssm_oracle_real_ex.restype = ctypes.c_int
            lib.ssm_oracle_complex.argtypes = [I64, I64, I64] + [P] * 6 + [I64, I64, ctypes.c_int] + [P] * 6
            lib.ssm_oracle_complex.restype = ctypes.c_int
            lib.ssm_oracle_complex_rtrl.argtypes = [I64, I64, I64] + [P] * 6 + [ctypes.c_int] + [P] * 4
            lib.ssm_oracle_complex_rtrl.restype = ctypes.c_int
            lib.ssm_oracle_pdssm.argtypes = ([I64] * 5 + [P] * 6 + [ctypes.c_double, ctypes.c_int] +
                                             [P] * 6)
            lib.ssm_oracle_pdssm.restype = ctypes.c_int
            lib.ssm_oracle_dtproj.argtypes = [I64, I64, I64] + [P] * 4
            lib.ssm_oracle_dtproj.restype = ctypes.c_int
            lib.ssm_oracle_dtproj_bwd.argtypes = [I64, I64, I64] + [P] * 6
            lib.ssm_oracle_dtproj_bwd.restype = ctypes.c_int
            lib.ssm_oracle_max_threads.argtypes = []
            lib.ssm_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().ssm_oracle_max_threads())


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _c128(a):
    return np.ascontiguousarray(a, dtype=np.complex128)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def real(x, delta_raw, A_log, Bm, Cm, Dskip, dy=None, chunk=128, d_range=None, threads=0,
         want_ckpt=False, zoh=False, h0=None, dhL=None):
    """Real-mode forward (and, if ``dy`` is given, backward) in float64.

    Shapes: x, delta_raw, dy [B,L,D]; Bm, Cm [B,L,N]; A_log [D,N]; Dskip [D]; h0, dhL [B,D,N].
    Returns a dict with y [B,L,D] and the final state hL [B,D,N] (and ckpt [B,ceil(L/chunk),D,N] if
    asked), plus dx, ddelta_raw [B,L,D], dA_log [D,N], dB, dC [B,L,N], dD [D] and dh0 [B,D,N] when
    ``dy`` is given.  ``zoh`` selects the zero-order-hold input term; ``h0`` is the initial state
    (default zero) and ``dhL`` the upstream gradient of the final state (default zero).  With
    ``d_range=(lo, hi)`` only channels lo..hi-1 are computed: other entries of the per-channel
    outputs are NaN and dB/dC are the sums over those channels only.
    """
    lib = _load()
    x, delta_raw, A_log, Bm, Cm, Dskip = map(_f64, (x, delta_raw, A_log, Bm, Cm, Dskip))
    B, L, D = x.shape
    N = A_log.shape[1]
    assert delta_raw.shape == (B, L, D) and Bm.shape == (B, L, N) and Cm.shape == (B, L, N)
    assert A_log.shape == (D, N) and Dskip.shape == (D,)
    lo, hi = (0, D) if d_range is None else (int(d_range[0]), int(d_range[1]))
    nC = (L + chunk - 1) // chunk
    if h0 is not None:
        h0 = _f64(h0)
        assert h0.shape == (B, D, N)
    if dhL is not None:
        dhL = _f64(dhL)
        assert dhL.shape == (B, D, N)
    out = {"y": np.full((B, L, D), np.nan), "hL": np.full((B, D, N), np.nan)}
    if want_ckpt:
        out["ckpt"] = np.full((B, nC, D, N), np.nan)
    if dy is not None:
        dy = _f64(dy)
        assert dy.shape == (B, L, D)
        out.update(dx=np.full((B, L, D), np.nan), ddelta_raw=np.full((B, L, D), np.nan),
                   dA_log=np.full((D, N), np.nan), dB=np.zeros((B, L, N)),
                   dC=np.zeros((B, L, N)), dD=np.full((D,), np.nan),
                   dh0=np.full((B, D, N), np.nan))
    rc = lib.ssm_oracle_real_ex(B, L, D, N, int(chunk), _ptr(x), _ptr(delta_raw), _ptr(A_log),
                                _ptr(Bm), _ptr(Cm), _ptr(Dskip), _ptr(dy), lo, hi, int(threads),
                                int(bool(zoh)), _ptr(h0), _ptr(dhL),
                                _ptr(out["y"]), _ptr(out.get("ckpt")), _ptr(out.get("dx")),
                                _ptr(out.get("ddelta_raw")), _ptr(out.get("dA_log")),
                                _ptr(out.get("dB")), _ptr(out.get("dC")), _ptr(out.get("dD")),
                                _ptr(out["hL"]), _ptr(out.get("dh0")))
    if rc != 0:
        raise RuntimeError("ssm_oracle_real failed (bad argument or out of memory)")
    return out


def complex_(u, r, phi, lam, omega, g=None, k_range=None, threads=0):
    """Complex-mode forward (and backward if ``g`` is given) in float64 / complex128.

    Shapes: u, g [B,L,K] complex; r, phi [B,L]; lam, omega [K].
    Returns h [B,L,K], and du [B,L,K], dr, dphi [B,L], dlambda, domega [K] when ``g`` is given.
    """
    lib = _load()
    u = _c128(u)
    r, phi, lam, omega = map(_f64, (r, phi, lam, omega))
    B, L, K = u.shape
    assert r.shape == (B, L) and phi.shape == (B, L) and lam.shape == (K,) and omega.shape == (K,)
    lo, hi = (0, K) if k_range is None else (int(k_range[0]), int(k_range[1]))
    out = {"h": np.full((B, L, K), np.nan, dtype=np.complex128)}
    if g is not None:
        g = _c128(g)
        assert g.shape == (B, L, K)
        out.update(du=np.full((B, L, K), np.nan, dtype=np.complex128), dr=np.zeros((B, L)),
                   dphi=np.zeros((B, L)), dlambda=np.full((K,), np.nan),
                   domega=np.full((K,), np.nan))
    rc = lib.ssm_oracle_complex(B, L, K, _ptr(u), _ptr(r), _ptr(phi), _ptr(lam), _ptr(omega),
                                _ptr(g), lo, hi, int(threads), _ptr(out["h"]),
                                _ptr(out.get("du")), _ptr(out.get("dr")), _ptr(out.get("dphi")),
                                _ptr(out.get("dlambda")), _ptr(out.get("domega")))
    if rc != 0:
        raise RuntimeError("ssm_oracle_complex failed (bad argument or out of memory)")
    return out


def complex_rtrl(u, r, phi, lam, omega, g, state=None, want_h=False, threads=0):
    """Complex-mode forward with exact structured RTRL: the state's sensitivities to lambda and
    omega are carried forward and the gradient of Re sum conj(g) h accumulates online.

    Shapes: u, g [B,L,K] complex; r, phi [B,L]; lam, omega [K]; state [B,3,K] complex holding
    (h, dh/dlambda, dh/domega) before the first step (default zero).  Returns a dict with
    dlambda, domega [K], state [B,3,K] (after the last step) and, if asked, h [B,L,K].
    """
    lib = _load()
    u, g = _c128(u), _c128(g)
    r, phi, lam, omega = map(_f64, (r, phi, lam, omega))
    B, L, K = u.shape
    assert g.shape == (B, L, K) and r.shape == (B, L) and phi.shape == (B, L)
    st = np.zeros((B, 3, K), dtype=np.complex128) if state is None else _c128(state).copy()
    assert st.shape == (B, 3, K)
    out = {"dlambda": np.full((K,), np.nan), "domega": np.full((K,), np.nan), "state": st}
    if want_h:
        out["h"] = np.full((B, L, K), np.nan, dtype=np.complex128)
    rc = lib.ssm_oracle_complex_rtrl(B, L, K, _ptr(u), _ptr(r), _ptr(phi), _ptr(lam),
                                     _ptr(omega), _ptr(g), int(threads), _ptr(out.get("h")),
                                     _ptr(st), _ptr(out["dlambda"]), _ptr(out["domega"]))
    if rc != 0:
        raise RuntimeError("ssm_oracle_complex_rtrl failed (bad argument)")
    return out


def pdssm(scores, dictionary, d, bt, h0=None, g=None, tau=1.0, threads=0):
    """Flash PD-SSM scan (hard selection forward, straight-through backward) in float64.

    Shapes: scores [B,L,H,K]; dictionary [K,N] int (row of the single 1 in each column of each
    dictionary matrix); d, bt, g [B,L,H,N]; h0 [B,H,N].  Returns h [B,L,H,N] and sel [B,L,H]
    (int32), plus dd, dbt [B,L,H,N], dscores [B,L,H,K], dh0 [B,H,N] when ``g`` is given.
    """
    lib = _load()
    scores, d, bt = _f64(scores), _f64(d), _f64(bt)
    dic = np.ascontiguousarray(dictionary, dtype=np.int32)
    B, L, H, K = scores.shape
    N = d.shape[-1]
    assert dic.shape == (K, N) and d.shape == (B, L, H, N) and bt.shape == (B, L, H, N)
    if h0 is not None:
        h0 = _f64(h0)
        assert h0.shape == (B, H, N)
    out = {"h": np.full((B, L, H, N), np.nan), "sel": np.full((B, L, H), -1, dtype=np.int32)}
    if g is not None:
        g = _f64(g)
        assert g.shape == (B, L, H, N)
        out.update(dd=np.full((B, L, H, N), np.nan), dbt=np.full((B, L, H, N), np.nan),
                   dscores=np.full((B, L, H, K), np.nan), dh0=np.full((B, H, N), np.nan))
    rc = lib.ssm_oracle_pdssm(B, L, H, N, K, _ptr(scores), _ptr(dic), _ptr(d), _ptr(bt), _ptr(h0),
                              _ptr(g), float(tau), int(threads), _ptr(out["h"]), _ptr(out["sel"]),
                              _ptr(out.get("dd")), _ptr(out.get("dbt")), _ptr(out.get("dscores")),
                              _ptr(out.get("dh0")))
    if rc != 0:
        raise RuntimeError("ssm_oracle_pdssm failed (bad argument or out of memory)")
    return out


def dtproj(u, w, bias=None, g=None):
    """Step-size projection delta_raw[m, d] = sum_r u[m, r] w[d, r] + bias[d] over the rows of u
    ([M, R] or [B, L, R]); with g = dL/d delta_raw also du, dw and dbias (see ssm_oracle.c)."""
    lib = _load()
    u = _f64(u)
    lead = u.shape[:-1]
    R = u.shape[-1]
    u2 = u.reshape(-1, R)
    w = _f64(w)
    D = w.shape[0]
    assert w.shape == (D, R)
    M = u2.shape[0]
    b = _f64(bias) if bias is not None else None
    out = np.empty((M, D))
    if lib.ssm_oracle_dtproj(M, D, R, _ptr(u2), _ptr(w), _ptr(b) if b is not None else None,
                             _ptr(out)) != 0:
        raise RuntimeError("ssm_oracle_dtproj failed")
    res = {"delta_raw": out.reshape(*lead, D)}
    if g is not None:
        g2 = _f64(g).reshape(M, D)
        du = np.empty((M, R))
        dw = np.empty((D, R))
        dbias = np.empty(D)
        if lib.ssm_oracle_dtproj_bwd(M, D, R, _ptr(u2), _ptr(w), _ptr(g2), _ptr(du), _ptr(dw),
                                     _ptr(dbias)) != 0:
            raise RuntimeError("ssm_oracle_dtproj_bwd failed")
        res.update(du=du.reshape(*lead, R), dw=dw, dbias=dbias)
    return res
