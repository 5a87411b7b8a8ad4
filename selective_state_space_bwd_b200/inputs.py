"""Seeded synthetic inputs for the selective scan, shared by the CUDA path and the oracle.

This module only draws random numbers and rounds them to the I/O precision; it contains none of
the scan's arithmetic.  Both sides of every parity test consume exactly the arrays returned
here (float32 holders; for bf16 workloads every value is already bf16-representable, so the
oracle's float64 upcast and the GPU's bf16 tensor hold the same numbers).

Workloads (value ranges follow the blog's step-size hygiene, "S3M 原理与工程实践" §5.2, and the
Phase Gradient Flow abstract's 128,000-step impulse-response benchmark):

* ``tiny``            B=1, L=256,    D=4,    N=4,  fp32
* ``mamba130m_layer`` B=8, L=2048,   D=1536, N=16, bf16
* ``stiff_impulse``   B=1, L=128000, D=1024, N=16, fp32 (unit impulse at t=0 plus noise, stiff A)
* ``mamba1p4b_layer`` B=4, L=8192,   D=4096, N=16, bf16
* ``mamba1p4b_layer_l2048`` the same with L=2048 (same grids and kernel instances: profiling)
* ``sparc_complex``   B=16, L=4096,  K=2048 complex modes (SPARC shared retention/phase control)
* ``sparc_complex_b4`` the same with B=4 (a quarter of the data: profiling captures)
* ``pdssm_l5120``     Flash PD-SSM scan: B=8, L=5120 (the sequence length of the Flash PD-SSM
                      throughput comparison), H=256 heads, N=16 states, K=8 dictionary matrices

Draw order (one ``numpy.random.default_rng(seed)`` stream, float32 draws): real mode
A_log (stiff only), delta_raw, x, Bm, Cm, Dskip, dy; complex mode lambda, omega, r, phi, u, g.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclass(frozen=True)
class RealWorkload:
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    chunk: int
    io: str
    kind: str  # "mamba" or "stiff"


@dataclass(frozen=True)
class ComplexWorkload:
    name: str
    batch: int
    seqlen: int
    modes: int
    chunk: int


WORKLOADS = {
    "tiny": RealWorkload("tiny", 1, 256, 4, 4, 128, F32, "mamba"),
    "mamba130m_layer": RealWorkload("mamba130m_layer", 8, 2048, 1536, 16, 128, BF16, "mamba"),
    "stiff_impulse": RealWorkload("stiff_impulse", 1, 128000, 1024, 16, 128, F32, "stiff"),
    "mamba1p4b_layer": RealWorkload("mamba1p4b_layer", 4, 8192, 4096, 16, 128, BF16, "mamba"),
    # a quarter of mamba1p4b_layer along L: the same grids and kernel instances (profiling captures)
    "mamba1p4b_layer_l2048": RealWorkload("mamba1p4b_layer_l2048", 4, 2048, 4096, 16, 128, BF16, "mamba"),
    "sparc_complex": ComplexWorkload("sparc_complex", 16, 4096, 2048, 128),
    "sparc_complex_b4": ComplexWorkload("sparc_complex_b4", 4, 4096, 2048, 128),
    # a quarter of sparc_complex along L with the same launch plan (profiling captures)
    "sparc_complex_l1024": ComplexWorkload("sparc_complex_l1024", 16, 1024, 2048, 128),
    "pdssm_l5120": None,  # filled below (PdWorkload is defined after this table)
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), returned as float32 in place."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    step = 1 << 24
    flat = u.reshape(-1)
    for s in range(0, flat.size, step):
        blk = flat[s:s + step]
        blk += np.uint32(0x7FFF) + ((blk >> np.uint32(16)) & np.uint32(1))
        blk &= np.uint32(0xFFFF0000)
    return a


def _inv_softplus(v: float) -> float:
    # log(expm1(v)): the raw value whose softplus is v (used only to set a sampling range)
    return math.log(math.expm1(v))


def real_inputs(batch, seqlen, dim, dstate, io=F32, kind="mamba", seed=0):
    """Draw one real-mode problem.  Returns a dict of float32 numpy arrays.

    kind="mamba": A_log[d,n] = log(n+1); softplus(delta_raw) spans [1e-3, 1e-1];
                  x, Bm, Cm, Dskip, dy ~ N(0,1).
    kind="stiff": A_log ~ U(log 0.5, log 50) so -exp(A_log) spans [-50, -0.5];
                  softplus(delta_raw) spans [1e-3, 1]; x = unit impulse at t=0 plus N(0, 1e-3).
    Shapes: x, delta_raw, dy [B,L,D]; Bm, Cm [B,L,N]; A_log [D,N]; Dskip [D].
    """
    rng = np.random.default_rng(seed)
    B, L, D, N = int(batch), int(seqlen), int(dim), int(dstate)
    if kind == "stiff":
        A_log = rng.uniform(math.log(0.5), math.log(50.0), size=(D, N)).astype(np.float32)
        dr_hi = _inv_softplus(1.0)
    elif kind == "mamba":
        A_log = np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (D, 1)).astype(np.float32)
        dr_hi = _inv_softplus(1e-1)
    else:
        raise ValueError(f"unknown workload kind {kind!r}")
    dr_lo = _inv_softplus(1e-3)
    delta_raw = rng.uniform(dr_lo, dr_hi, size=(B, L, D)).astype(np.float32)
    if kind == "stiff":
        x = rng.standard_normal((B, L, D), dtype=np.float32)
        x *= np.float32(1e-3)
        if L > 0:
            x[:, 0, :] += np.float32(1.0)
    else:
        x = rng.standard_normal((B, L, D), dtype=np.float32)
    Bm = rng.standard_normal((B, L, N), dtype=np.float32)
    Cm = rng.standard_normal((B, L, N), dtype=np.float32)
    Dskip = rng.standard_normal((D,), dtype=np.float32)
    dy = rng.standard_normal((B, L, D), dtype=np.float32)
    out = dict(x=x, delta_raw=delta_raw, A_log=A_log, Bm=Bm, Cm=Cm, Dskip=Dskip, dy=dy)
    if io == BF16:
        for k in ("x", "delta_raw", "Bm", "Cm", "dy"):
            out[k] = round_to_bf16(out[k])
    elif io != F32:
        raise ValueError(f"unknown io dtype {io!r}")
    return out


def dtproj_inputs(batch, seqlen, dim, rank, seed=0):
    """Draw the step-size projection of one real-mode problem (bf16 I/O).

    u ~ N(0,1) [B,L,R] (the low-rank per-token input), w ~ N(0, 1/(4R)) [D,R], bias ~ U(lo, hi)
    [D] with lo, hi the raw values whose softplus is 2e-3 and 5e-2, so that u w^T + bias (spread
    ~0.5 about the bias) keeps softplus(delta_raw) near the workload's [1e-3, 1e-1]; the upstream
    gradient ddelta_raw ~ N(0,1) [B,L,D].  u, w, ddelta_raw are rounded to bf16; bias is fp32.
    """
    rng = np.random.default_rng(seed)
    B, L, D, R = int(batch), int(seqlen), int(dim), int(rank)
    u = round_to_bf16(rng.standard_normal((B, L, R), dtype=np.float32))
    w = round_to_bf16((rng.standard_normal((D, R)) / (2.0 * math.sqrt(R))).astype(np.float32))
    bias = rng.uniform(_inv_softplus(2e-3), _inv_softplus(5e-2), size=(D,)).astype(np.float32)
    g = round_to_bf16(rng.standard_normal((B, L, D), dtype=np.float32))
    return dict(u=u, w=w, bias=bias, g=g)


def complex_inputs(batch, seqlen, modes, seed=0):
    """Draw one complex-mode problem (SPARC-style shared control).

    lambda_k = exp(U(log 1e-3, 0)); omega_k ~ U(0, pi); r, phi ~ N(0,1) per (b,t);
    u, g ~ CN(0,1) with independent real and imaginary parts of variance 1/2.
    Shapes: u, g [B,L,K] complex64; r, phi [B,L]; lambda, omega [K].
    """
    rng = np.random.default_rng(seed)
    B, L, K = int(batch), int(seqlen), int(modes)
    lam = np.exp(rng.uniform(math.log(1e-3), 0.0, size=(K,))).astype(np.float32)
    omega = rng.uniform(0.0, math.pi, size=(K,)).astype(np.float32)
    r = rng.standard_normal((B, L), dtype=np.float32)
    phi = rng.standard_normal((B, L), dtype=np.float32)
    s = np.float32(math.sqrt(0.5))
    u = np.empty((B, L, K), dtype=np.complex64)
    u.real = rng.standard_normal((B, L, K), dtype=np.float32) * s
    u.imag = rng.standard_normal((B, L, K), dtype=np.float32) * s
    g = np.empty((B, L, K), dtype=np.complex64)
    g.real = rng.standard_normal((B, L, K), dtype=np.float32) * s
    g.imag = rng.standard_normal((B, L, K), dtype=np.float32) * s
    return dict(u=u, r=r, phi=phi, lam=lam, omega=omega, g=g)


def workload_inputs(name, seed=0):
    w = WORKLOADS[name]
    if isinstance(w, ComplexWorkload):
        return complex_inputs(w.batch, w.seqlen, w.modes, seed)
    if type(w).__name__ == "PdWorkload":
        return pdssm_inputs(w.batch, w.seqlen, w.heads, w.nstate, w.ndict, seed)
    return real_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.io, w.kind, seed)


def pdssm_inputs(batch, seqlen, heads, nstate, ndict, seed=0):
    """Draw one Flash PD-SSM problem.

    scores ~ N(0,1) [B,L,H,K]; dictionary: K random maps of the N columns to rows (each column of
    each matrix holds a single 1), [K,N] int32; d ~ U(0.3, 0.9) [B,L,H,N] (so every transition
    shrinks the state's 1-norm); bt, g ~ N(0,1) [B,L,H,N]; h0 ~ N(0,1) [B,H,N].
    """
    rng = np.random.default_rng(seed)
    B, L, H, N, K = int(batch), int(seqlen), int(heads), int(nstate), int(ndict)
    dictionary = rng.integers(0, N, size=(K, N), dtype=np.int32)
    scores = rng.standard_normal((B, L, H, K), dtype=np.float32)
    d = rng.uniform(0.3, 0.9, size=(B, L, H, N)).astype(np.float32)
    bt = rng.standard_normal((B, L, H, N), dtype=np.float32)
    g = rng.standard_normal((B, L, H, N), dtype=np.float32)
    h0 = rng.standard_normal((B, H, N), dtype=np.float32)
    return dict(scores=scores, dictionary=dictionary, d=d, bt=bt, g=g, h0=h0)


@dataclass(frozen=True)
class PdWorkload:
    name: str
    batch: int
    seqlen: int
    heads: int
    nstate: int
    ndict: int


WORKLOADS["pdssm_l5120"] = PdWorkload("pdssm_l5120", 8, 5120, 256, 16, 8)
# a quarter of pdssm_l5120 along L with the same launch plan (profiling captures)
WORKLOADS["pdssm_l1280"] = PdWorkload("pdssm_l1280", 8, 1280, 256, 16, 8)
