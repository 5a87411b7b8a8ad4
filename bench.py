#!/usr/bin/env python
"""Throughput of the selective scan's forward + exact backward on B200.

One step = ssm_scan_fwd + ssm_scan_bwd over one batch of the workload (inputs resident in HBM),
plus, with more than one rank, the data-parallel all-reduce of the parameter gradients
(dA_log, dD).  Each rank owns a full batch of the workload (weak scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Rank 0 prints one JSON line.  ``value`` is state-updates/s over all ranks (B*L*D*N per rank per
step), device-timed with CUDA events, max over ranks; L2 is flushed (a 256 MiB write, then a
256 MiB read that evicts the written lines) before every timed step, outside the events.  ``e2e``
is the same metric through the same calls with the inputs copied in from pinned host memory and
every output copied back inside the timed region.
``--impl reference`` times the float64 CPU oracle on the host cores instead (bounded sample).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd scan state-updates/s (B·L·D·N/s); achieved HBM GB/s vs B200 peak"
UNIT = "state-updates/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mamba1p4b_layer",
                    help="default: the largest single-GPU real workload (B=4, L=8192, D=4096, N=16, bf16)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seg-chunks", type=int, default=0)
    ap.add_argument("--zoh", action="store_true",
                    help="zero-order-hold input term instead of Euler (ssm_scan_*_ex)")
    ap.add_argument("--fused-sums", action="store_true",
                    help="real backward with SSM_FUSED_SUMS: dB/dC sums inside the scan kernel "
                         "(cooperative launches), less DRAM traffic, no reduction launch")
    ap.add_argument("--rtrl", action="store_true",
                    help="complex workloads: time exact structured RTRL (one forward pass that "
                         "accumulates dlambda, domega online) instead of fwd + bwd")
    ap.add_argument("--ckpt", action="store_true",
                    help="complex workloads: the forward also writes chunk checkpoints and the "
                         "backward recomputes from them (ssm_scan_complex_bwd) instead of reading "
                         "the stored trajectory (ssm_scan_complex_bwd_traj)")
    ap.add_argument("--state", action="store_true",
                    help="pass an initial state h0 and an upstream final-state gradient dhL")
    ap.add_argument("--dtproj", type=int, default=0, metavar="R",
                    help="bf16 real workloads: compute delta_raw every step with the rank-R step-size "
                         "projection (ssm_dtproj_fwd) and its gradient (ssm_dtproj_bwd)")
    ap.add_argument("--memory-curve", action="store_true",
                    help="peak device memory of fwd+bwd vs L for the stiff workload's shape")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# FP32-pipe lane operations per state update (an FMA counts as one), the minimum the arithmetic
# of the method needs, with per-(t, d) and per-(t, n) terms (O(1/N), O(1/D)) left out:
#   forward:  delta*A'; u*B; h = a*h + u*B; y += C*h                                      -> 4
#   backward: recompute delta*A', p = a*h_prev, h = p + u*B (3); g = C*dy + v; v = a*g;
#             dB += u*g; dC += dy*h; q = g*p; dA += delta*q; sum A*q; sum g*B (8)           -> 11
# plus one exp2 (MUFU) per update in each direction.
FWD_OPS_PER_UPDATE = 4
BWD_OPS_PER_UPDATE = 11
# zero-order hold adds, per update: phi = (a - 1) / A (2) and x phi (1) forward; in the backward
# the same 2 in the recompute, psi = (delta a - phi) / A (3), g B x psi into dA (2), sum g a B (1)
ZOH_FWD_OPS_PER_UPDATE = 7
ZOH_BWD_OPS_PER_UPDATE = 19
SMS, FP32_LANES_PER_SM = 148, 128
# MUFU ex2 results per SM per clock (measured with a microbenchmark on this B200), and the exp2
# the kernels evaluate per update: the forward one, the backward two (the chunk walk that finds
# each window's start state, and the window's own recompute)
MUFU_EX2_PER_SM = 16
FWD_EXP2_PER_UPDATE, BWD_EXP2_PER_UPDATE = 1, 2


def alu_peak_tops():
    """FP32-pipe lane operations per second at the maximum SM clock: 148 SMs x 128 lanes x f."""
    mhz = 1965.0
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        mhz = float(json.load(open(p)).get("sm_max_mhz", mhz))
    return SMS * FP32_LANES_PER_SM * mhz * 1e6 / 1e12, mhz


def clock_roofs(clk, achieved_tops, updates_per_s, exp2_per_update):
    """The FP32-pipe and MUFU roofs at the SM clock sampled during the timed region (the fixed
    peak above assumes the maximum clock), and the fractions of them achieved."""
    mhz = clk.get("sm_mhz") if clk else None
    if not mhz:
        return {}
    fp32 = SMS * FP32_LANES_PER_SM * mhz * 1e6 / 1e12
    mufu = SMS * MUFU_EX2_PER_SM * mhz * 1e6  # exp2 per second
    return {"sampled_sm_mhz": mhz, "peak_at_sampled_clock": fp32,
            "frac_at_sampled_clock": achieved_tops / fp32,
            "mufu_ex2_per_s_at_sampled_clock": mufu,
            "mufu_frac_at_sampled_clock": updates_per_s * exp2_per_update / mufu}


def algorithmic_bytes(w):
    """Minimum bytes the method moves per step (fwd + bwd), split by call."""
    from selective_state_space_bwd_b200 import inputs as gen
    s = 2 if w.io == gen.BF16 else 4
    E = w.batch * w.seqlen * w.dim
    BLN = w.batch * w.seqlen * w.dstate
    nC = -(-w.seqlen // w.chunk)
    ck = w.batch * nC * w.dim * w.dstate * 4
    fwd = 3 * E * s + 2 * BLN * s + ck           # x, delta_raw in; y out; Bm, Cm in; ckpt out
    bwd = 5 * E * s + 4 * BLN * s + ck           # x, delta_raw, dy in; dx, ddelta_raw out;
    return fwd, bwd                              # Bm, Cm in; dB, dC out; ckpt in


def dtproj_algorithmic(w, R):
    """Minimum bytes of the step-size projection's forward (u, w read, bias read, delta_raw
    written; bf16 except the fp32 bias) and backward (g = ddelta_raw read once, u and w read, du
    written bf16, dw and dbias written fp32), and the FLOPs of one of its GEMMs (2 M D R)."""
    M, D = w.batch * w.seqlen, w.dim
    fwd = 2 * M * R + 2 * D * R + 4 * D + 2 * M * D
    bwd = 2 * M * D + 2 * M * R + 2 * D * R + 2 * M * R + 4 * D * R + 4 * D
    return fwd, bwd, 2 * M * D * R


def e2e_pipelined(torch, dev, stream, host, sets, compute, outputs, steps, world, dist):
    """Seconds (max over ranks) for `steps` end-to-end steps.  Every step copies its inputs from
    pinned host memory (`host` into set["d"]) on one copy stream, computes on `stream`, and copies
    `outputs(set)` back into pinned host buffers on another; the steps alternate between the two
    device buffer sets, so one step's copies run beside the next step's compute while every step
    still moves all its bytes.  Returns (seconds, h2d bytes per step, d2h bytes per step)."""
    hout = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in outputs(sets[0]).items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in hout.values())
    s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(nsteps, start_event=None):
        if start_event is not None:
            s_h2d.wait_event(start_event)
        for k in range(nsteps):
            i = k % 2
            bs = sets[i]
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_event(ev_done[i])  # set i's inputs are free once its last compute ended
                for key, v in host.items():
                    bs["d"][key].copy_(v, non_blocking=True)
                ev_in[i].record(s_h2d)
            stream.wait_event(ev_in[i])
            stream.wait_event(ev_out[i])  # set i's outputs were copied back
            compute(bs)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_done[i])
                for key, v in outputs(bs).items():
                    hout[key].copy_(v, non_blocking=True)
                ev_out[i].record(s_d2h)
        stream.wait_event(ev_out[(nsteps - 1) % 2])

    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    run(steps, start_event=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    t = torch.tensor([e0.elapsed_time(e1) / 1e3], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t), h2d, d2h


E2E_OVERLAP = ("two buffer sets; each step's host-to-device and device-to-host copies run on their "
               "own streams beside the next step's compute")


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML every 1 ms while the timed region runs
    (a background thread), so even a timed region of a few tens of milliseconds gets tens of
    samples.  The GPU is found by its PCI bus id (falling back to the device index).  The raw
    samples go to clocks_rank<i>.csv in $SSM_BENCH_CLOCKS_DIR (default: the system temp dir)."""

    PERIOD_S = 0.001
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.handle = None
        self.samples = []
        import tempfile
        out = os.environ.get("SSM_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out, f"clocks_rank{index}.csv")

    def _open(self):
        import pynvml as nv
        nv.nvmlInit()
        h = None
        try:
            import torch
            pr = torch.cuda.get_device_properties(self.index)
            bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            h = nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            h = None
        return nv, (h if h is not None else nv.nvmlDeviceGetHandleByIndex(self.index))

    def start(self):
        import threading
        try:
            self.nv, self.handle = self._open()
            self.smax = float(self.nv.nvmlDeviceGetMaxClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
        except Exception:
            self.handle = None
            return
        nv = self.nv
        bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        self.stop_flag = threading.Event()

        def run():
            while not self.stop_flag.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1e3
                except Exception:
                    break
                self.samples.append((time.time(), float(mhz), pw, [bool(rs & b) for b in bits]))
                time.sleep(self.PERIOD_S)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        self.stop_flag.set()
        self.thread.join(timeout=5)
        reasons = set()
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            with open(self.path, "w") as fh:
                fh.write("time_s,sm_mhz,power_w," + ",".join(self.NAMES) + "\n")
                for t, mhz, pw, act in self.samples:
                    fh.write(f"{t:.4f},{mhz:.0f},{pw:.1f}," + ",".join(str(int(a)) for a in act) + "\n")
        except OSError:
            pass
        for _, _, _, act in self.samples:
            reasons.update(n for n, a in zip(self.NAMES, act) if a)
        sm = [s[1] for s in self.samples]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "reasons": sorted(reasons), "samples": len(sm), "sampler": "NVML, 1 ms period",
                "power_w_max": max((s[2] for s in self.samples), default=None)}


def oracle_sample(w, inp, budget_s=(10.0, 30.0), zoh=False):
    """Time the float64 oracle on the host cores: whole batch rows of the workload, repeated
    until about budget_s[0] seconds of work (stops before budget_s[1])."""
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    rows = 0
    t_total = 0.0
    b = 0
    while t_total < budget_s[0]:
        sl = slice(b, b + 1)
        t0 = time.perf_counter()
        oracle.real(inp["x"][sl], inp["delta_raw"][sl], inp["A_log"], inp["Bm"][sl], inp["Cm"][sl],
                    inp["Dskip"], inp["dy"][sl], chunk=w.chunk, threads=threads, zoh=zoh)
        dt = time.perf_counter() - t0
        t_total += dt
        rows += 1
        b = (b + 1) % w.batch
        if t_total + dt > budget_s[1]:
            break
    upd = rows * w.seqlen * w.dim * w.dstate
    return {"value": upd / t_total, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} batch-row runs, cycling over the {w.batch} rows of {w.name} "
                      f"(L={w.seqlen}, D={w.dim}, N={w.dstate}), fwd+bwd in float64, {t_total:.1f} s"}


def code_digest(path):
    """sha256 of a C++/CUDA source's code: `//` comments, surrounding blanks and empty lines
    dropped, so that an edit of the comments alone keeps a traffic record valid."""
    import hashlib
    lines = []
    for line in open(path, encoding="utf-8").read().splitlines():
        code = line.split("//", 1)[0].strip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def measured_traffic(call, kernel_file, workload):
    """DRAM bytes per launch of `call` (its kernels summed) on `workload`, from the committed ncu
    capture records, if that capture was taken on the current code of `kernel_file`; else None.
    A record captured on a smaller case of the same launch plan carries the factor that scales
    it to the full workload's units."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        recs = json.load(open(p))["records"]
        sha = code_digest(os.path.join(ROOT, "selective_state_space_bwd_b200", "csrc", kernel_file))
        for rec in recs:
            if (rec["workload"] == workload and rec["call"] == call and rec["source"] == kernel_file
                    and rec["code_sha256"] == sha):
                return float(rec["dram_bytes_per_launch"])
        return None
    except (OSError, ValueError, KeyError, TypeError):
        return None


def memory_curve():
    """Peak device memory of one fwd+bwd at the stiff workload's width (B=1, D=1024, N=16,
    fp32, T=128) for growing L, minus the inputs and outputs themselves."""
    import torch
    from selective_state_space_bwd_b200 import build, ssm_scan as S
    build.build()
    dev = torch.device("cuda", 0)
    B, D, N, T = 1, 1024, 16, 128
    rows = []
    for L in (8000, 16000, 32000, 64000, 128000):
        torch.cuda.empty_cache()
        x = torch.randn(B, L, D, device=dev)
        dr = torch.rand(B, L, D, device=dev) * 7.4 - 6.9
        dy = torch.randn(B, L, D, device=dev)
        A_log = torch.rand(D, N, device=dev) * 4.6 - 0.7
        Bm, Cm = torch.randn(B, L, N, device=dev), torch.randn(B, L, N, device=dev)
        Dskip = torch.randn(D, device=dev)
        y = torch.empty_like(x)
        out = dict(dx=torch.empty_like(x), ddelta_raw=torch.empty_like(x),
                   dA_log=torch.empty_like(A_log), dB=torch.empty_like(Bm), dC=torch.empty_like(Cm),
                   dD=torch.empty_like(Dskip))
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        y, ck = S.ssm_scan_fwd(x, dr, A_log, Bm, Cm, Dskip, chunk=T, y=y)
        S.ssm_scan_bwd(x, dr, A_log, Bm, Cm, Dskip, ck, dy, chunk=T, out=out)
        torch.cuda.synchronize()
        peak = torch.cuda.max_memory_allocated() - base
        shape = S.real_shape(B, L, D, N, T, S.SSM_F32)
        rows.append({"L": L, "extra_peak_bytes": peak,
                     "checkpoint_bytes": S.checkpoint_bytes(shape),
                     "fwd_workspace_bytes": S.workspace_bytes(shape, False),
                     "bwd_workspace_bytes": S.workspace_bytes(shape, True),
                     "every_state_bytes": L * D * N * 4})
        del x, dr, dy, Bm, Cm, y, out, ck
    print(json.dumps({"metric": "peak device memory beyond inputs/outputs, fwd+bwd",
                      "shape": {"batch": B, "dim": D, "dstate": N, "chunk": T, "io": "f32"},
                      "curve": rows}), flush=True)


L2_NOTE = ("flushed (256 MiB write, then a 256 MiB read that evicts the written lines) before "
           "every timed step")


class L2Flush:
    """Before each timed step, outside its events: a write of a buffer twice the L2 evicts every
    input, and a read of a second such buffer then evicts the written (dirty) lines, so that their
    write-back to DRAM does not land on the first kernel of the step."""

    def __init__(self, dev):
        import torch
        self.wr = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.rd = torch.zeros((256 << 20) // 4, dtype=torch.float32, device=dev)
        self.acc = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.wr.zero_()
        torch.sum(self.rd, dim=(0,), out=self.acc)


def real_config(args, w, world):
    """The workload a real-mode line measures (both arms print the same dict)."""
    c = {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
         "dstate": w.dstate, "chunk": w.chunk, "io": w.io,
         "discretization": "zoh" if args.zoh else "euler",
         "dbc_sums": "fused into the scan kernel (SSM_FUSED_SUMS)" if args.fused_sums else "reduction kernel",
         "initial_state": bool(args.state), "state": "fp32", "l2": L2_NOTE,
         "parallelism": f"dp{world} (weak: one full batch per rank; dA_log/dD all-reduced)"
                        if world > 1 else "single GPU"}
    if args.dtproj:
        c["dt_rank"] = args.dtproj
    return c


def complex_config(args, w, world):
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
            "modes": w.modes, "chunk": w.chunk, "io": "complex64",
            "training": "rtrl (online, forward only)" if args.rtrl else "bptt (fwd + bwd)",
            "backward": ("from chunk checkpoints (ssm_scan_complex_bwd)" if args.ckpt
                         else "from the stored trajectory (ssm_scan_complex_bwd_traj)"),
            "l2": L2_NOTE,
            "parallelism": f"dp{world} (weak: one full batch per rank; dlambda/domega all-reduced)"
                           if world > 1 else "single GPU"}


def pdssm_config(args, w, world):
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "heads": w.heads,
            "nstate": w.nstate, "ndict": w.ndict, "tau": 1.0, "l2": L2_NOTE,
            "parallelism": f"dp{world} (weak: one full batch per rank, no exchange)"
                           if world > 1 else "single GPU"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from selective_state_space_bwd_b200 import inputs as gen
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    cplx = isinstance(w, gen.ComplexWorkload)
    if isinstance(w, gen.PdWorkload):
        return run_reference_pdssm(args, w)
    if cplx:
        inp = gen.complex_inputs(1, w.seqlen, w.modes, seed=0)
        upd = w.seqlen * w.modes
    else:
        inp = gen.real_inputs(1, w.seqlen, w.dim, w.dstate, w.io, w.kind, seed=0)
        upd = w.seqlen * w.dim * w.dstate
    times = []
    for k in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if cplx:
            oracle.complex_(inp["u"], inp["r"], inp["phi"], inp["lam"], inp["omega"], inp["g"],
                            threads=threads)
        else:
            oracle.real(inp["x"], inp["delta_raw"], inp["A_log"], inp["Bm"], inp["Cm"],
                        inp["Dskip"], inp["dy"], chunk=w.chunk, threads=threads, zoh=args.zoh)
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = upd * len(times) / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, shapes of the workload)",
            "config": (complex_config if cplx else real_config)(args, w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"1 of {w.batch} batch rows of {w.name} per step (fwd + "
                                       f"bwd in float64 on the host cores; no L2 flush)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def complex_algorithmic_bytes(w, ckpt=False):
    """Minimum bytes of one complex fwd + bwd (8 B per complex64 element, 4 B per real one).
    From the stored trajectory: the forward reads u and writes h, the backward reads h and g and
    writes du.  From chunk checkpoints (ckpt): the forward reads u and writes the checkpoints, the
    backward reads them, u and g and writes du.  Both read r and phi; the backward writes dr and
    dphi."""
    BLK, BL = w.batch * w.seqlen * w.modes, w.batch * w.seqlen
    if ckpt:
        ck = w.batch * (-(-w.seqlen // w.chunk)) * w.modes * 8
        return 8 * BLK + 8 * BL + ck, 24 * BLK + 16 * BL + ck
    return 16 * BLK + 8 * BL, 24 * BLK + 16 * BL


def oracle_sample_complex(w, inp, budget_s=(10.0, 30.0), rtrl=False):
    """Time the float64 oracle's complex mode on whole batch rows (about budget_s[0] seconds)."""
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    rows, t_total, b = 0, 0.0, 0
    while t_total < budget_s[0]:
        sl = slice(b, b + 1)
        t0 = time.perf_counter()
        if rtrl:
            oracle.complex_rtrl(inp["u"][sl], inp["r"][sl], inp["phi"][sl], inp["lam"],
                                inp["omega"], inp["g"][sl], threads=threads)
        else:
            oracle.complex_(inp["u"][sl], inp["r"][sl], inp["phi"][sl], inp["lam"], inp["omega"],
                            inp["g"][sl], threads=threads)
        dt = time.perf_counter() - t0
        t_total += dt
        rows += 1
        b = (b + 1) % w.batch
        if t_total + dt > budget_s[1]:
            break
    upd = rows * w.seqlen * w.modes
    return {"value": upd / t_total, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} batch row(s) of {w.name} (L={w.seqlen}, K={w.modes}), "
                      f"{'RTRL' if rtrl else 'fwd+bwd'} in float64 / complex128, {t_total:.1f} s"}


def main_complex(args, w):
    """The complex-mode (shared retention/phase) scan: ssm_scan_complex_fwd + _bwd per step."""
    import torch
    import torch.distributed as dist
    from selective_state_space_bwd_b200 import build, dp, ssm_scan as S
    from selective_state_space_bwd_b200 import inputs as gen

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    S.lib()
    inp = gen.complex_inputs(w.batch, w.seqlen, w.modes, seed=rank)
    host = {k: torch.from_numpy(v).pin_memory() for k, v in inp.items()}
    d = {k: v.to(dev) for k, v in host.items()}
    shape = S.complex_shape(w.batch, w.seqlen, w.modes, w.chunk, args.seg_chunks)
    h = torch.empty_like(d["u"])
    out = dict(du=torch.empty_like(d["g"]), dr=torch.empty_like(d["r"]),
               dphi=torch.empty_like(d["phi"]), dlambda=torch.empty_like(d["lam"]),
               domega=torch.empty_like(d["omega"]))
    wsf = torch.empty(S.complex_workspace_bytes(shape, False), dtype=torch.uint8, device=dev)
    wsb = torch.empty(S.complex_workspace_bytes(shape, True), dtype=torch.uint8, device=dev)
    gbuf = torch.empty(2 * w.modes, dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    if args.rtrl:
        out = dict(dlambda=out["dlambda"], domega=out["domega"])
        wsr = torch.empty(S.complex_rtrl_workspace_bytes(shape), dtype=torch.uint8, device=dev)

    nC = -(-w.seqlen // w.chunk)
    ck = (torch.empty((w.batch, nC, w.modes), dtype=torch.complex64, device=dev)
          if args.ckpt else None)
    sets = [dict(d=d, h=h, ck=ck, out=out)]

    def fwd(bs=None):
        bs = bs or sets[0]
        dd, hh, oo = bs["d"], bs["h"], bs["out"]
        if args.rtrl:  # the whole RTRL pass: trajectory sensitivities and online gradient
            S.ssm_scan_complex_rtrl(dd["u"], dd["r"], dd["phi"], dd["lam"], dd["omega"], dd["g"],
                                    chunk=w.chunk, out=oo, ws=wsr, stream=stream)
        else:
            S.ssm_scan_complex_fwd(dd["u"], dd["r"], dd["phi"], dd["lam"], dd["omega"], chunk=w.chunk,
                                   seg_chunks=args.seg_chunks, h=hh, ckpt=bs["ck"], ws=wsf,
                                   stream=stream)

    def bwd(bs=None):
        bs = bs or sets[0]
        dd, hh, oo = bs["d"], bs["h"], bs["out"]
        if args.rtrl:
            return
        if args.ckpt:  # recompute every chunk from its checkpoint
            S.ssm_scan_complex_bwd(dd["u"], dd["r"], dd["phi"], dd["lam"], dd["omega"], bs["ck"],
                                   dd["g"], chunk=w.chunk, seg_chunks=args.seg_chunks, out=oo,
                                   ws=wsb, stream=stream)
        else:  # read h_{t-1} from the stored trajectory
            S.ssm_scan_complex_bwd_traj(hh, dd["r"], dd["phi"], dd["lam"], dd["omega"], dd["g"],
                                        chunk=w.chunk, seg_chunks=args.seg_chunks, out=oo, ws=wsb,
                                        stream=stream)

    def allreduce(bs=None):
        oo = (bs or sets[0])["out"]
        if world > 1:  # dlambda, domega sum over the batch rows of every rank
            dp.allreduce_grads([oo["dlambda"], oo["domega"]], buf=gbuf)

    for _ in range(max(3, args.warmup)):
        fwd(); bwd(); allreduce()
    torch.cuda.synchronize()
    if S.ssm_scan_status(wsr if args.rtrl else wsb) != 0 or S.ssm_scan_status(wsf) != 0:
        raise SystemExit("device status word reports a non-finite state")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for k in range(args.steps):
        flush()
        e = ev[k]
        e[0].record(stream); fwd(); e[1].record(stream); bwd(); e[2].record(stream)
        allreduce(); e[3].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    t_fwd = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_bwd = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_step = sum(e[0].elapsed_time(e[3]) for e in ev) / 1e3
    tt = torch.tensor([t_step, t_fwd, t_bwd], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    t_step, t_fwd, t_bwd = tt.tolist()

    sets.append(dict(d={k: torch.empty_like(v) for k, v in d.items()}, h=torch.empty_like(h),
                     ck=torch.empty_like(ck) if ck is not None else None,
                     out={k: torch.empty_like(v) for k, v in out.items()}))

    def compute(bs):
        fwd(bs); bwd(bs); allreduce(bs)

    def outputs(bs):  # the RTRL pass returns only dlambda, domega
        return dict(bs["out"]) if args.rtrl else dict(h=bs["h"], **bs["out"])

    t_e2e, h2d, d2h = e2e_pipelined(torch, dev, stream, host, sets, compute, outputs, args.steps,
                                    world, dist)

    upd_rank = w.batch * w.seqlen * w.modes
    value = world * upd_rank * args.steps / t_step
    hbm, peak_kind = peaks()
    fb, bb = complex_algorithmic_bytes(w, ckpt=args.ckpt)
    if args.rtrl:  # u and g read (8 B each per update), r and phi read (4 B each per (b, t))
        fb, bb = 16 * w.batch * w.seqlen * w.modes + 8 * w.batch * w.seqlen, 0
    bwd_gbs = bb / (t_bwd / args.steps) / 1e9 if bb else 0.0
    fwd_gbs = fb / (t_fwd / args.steps) / 1e9
    launches = (S.complex_kernel_launches(shape, 0) +
                S.complex_kernel_launches(shape, 1 if args.ckpt else 2)) * args.steps
    if args.rtrl:
        launches = 2 * args.steps
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_step / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "c64",
            "data": "synthetic (seeded generator, workload value distributions)",
            "config": complex_config(args, w, world),
            "roofline": ({"bound": "hbm", "kernel": "ssm_scan_complex_rtrl call (cplx_rtrl_kernel "
                          "+ reduction over the batch)", "achieved": fwd_gbs, "peak": hbm,
                          "unit": "GB/s", "frac": fwd_gbs / hbm, "peak_kind": peak_kind,
                          "algorithmic_bytes_per_launch": fb,
                          "traffic": measured_traffic("ssm_scan_complex_rtrl", "complex_scan.cu",
                                                      w.name)} if args.rtrl else
                         {"bound": "hbm",
                          "kernel": ("ssm_scan_complex_bwd call (cplx_bwd_ckpt_kernel + reductions)"
                                     if args.ckpt else "ssm_scan_complex_bwd_traj call "
                                     "(cplx_bwd_kernel + reductions)"),
                          "achieved": bwd_gbs, "peak": hbm, "unit": "GB/s",
                          "frac": bwd_gbs / hbm, "peak_kind": peak_kind,
                          "algorithmic_bytes_per_launch": bb,
                          "traffic": measured_traffic("ssm_scan_complex_bwd" if args.ckpt else
                                                      "ssm_scan_complex_bwd_traj",
                                                      "complex_scan.cu", w.name)}),
            "hbm_frac_fwd": fwd_gbs / hbm, "hbm_frac_bwd": bwd_gbs / hbm,
            "ms_fwd": 1e3 * t_fwd / args.steps, "ms_bwd": 1e3 * t_bwd / args.steps,
            "e2e": {"value": world * upd_rank * args.steps / t_e2e, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": E2E_OVERLAP},
            "gpu_launches": launches,
            "clocks": clk,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = oracle_sample_complex(w, inp, rtrl=args.rtrl)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def pdssm_algorithmic_bytes(w):
    """Minimum bytes of one Flash PD-SSM fwd + bwd.  Forward: scores, d, bt read; h, sel written.
    Backward: scores, d, h, sel, g read; dd, dbt, dscores written (fp32; sel int32)."""
    BLH = w.batch * w.seqlen * w.heads
    upd = BLH * w.nstate
    return 12 * upd + (4 * w.ndict + 4) * BLH, 20 * upd + (8 * w.ndict + 4) * BLH


def oracle_sample_pdssm(w, inp, budget_s=(10.0, 30.0)):
    """Time the float64 oracle's Flash PD-SSM fwd + bwd on whole batch rows."""
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    rows, t_total, b = 0, 0.0, 0
    while t_total < budget_s[0]:
        sl = slice(b, b + 1)
        t0 = time.perf_counter()
        oracle.pdssm(inp["scores"][sl], inp["dictionary"], inp["d"][sl], inp["bt"][sl],
                     inp["h0"][sl], inp["g"][sl], tau=1.0, threads=threads)
        dt = time.perf_counter() - t0
        t_total += dt
        rows += 1
        b = (b + 1) % w.batch
        if t_total + dt > budget_s[1]:
            break
    upd = rows * w.seqlen * w.heads * w.nstate
    return {"value": upd / t_total, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} batch row(s) of {w.name} (L={w.seqlen}, H={w.heads}, "
                      f"N={w.nstate}, K={w.ndict}), fwd+bwd in float64, {t_total:.1f} s"}


def main_pdssm(args, w):
    """Flash PD-SSM: ssm_pdssm_fwd + ssm_pdssm_bwd per step.  Batch rows are independent and no
    parameter gradient is summed, so ranks exchange nothing but the timing."""
    import torch
    import torch.distributed as dist
    from selective_state_space_bwd_b200 import build, ssm_scan as S
    from selective_state_space_bwd_b200 import inputs as gen

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    S.lib()
    inp = gen.pdssm_inputs(w.batch, w.seqlen, w.heads, w.nstate, w.ndict, seed=rank)
    host = {k: torch.from_numpy(v).pin_memory() for k, v in inp.items()}
    d = {k: v.to(dev) for k, v in host.items()}
    h = torch.empty_like(d["d"])
    sel = torch.empty((w.batch, w.seqlen, w.heads), dtype=torch.int32, device=dev)
    out = dict(dd=torch.empty_like(d["d"]), dbt=torch.empty_like(d["d"]),
               dscores=torch.empty_like(d["scores"]), dh0=torch.empty_like(d["h0"]))
    shape = S.pdssm_shape(w.batch, w.seqlen, w.heads, w.nstate, w.ndict)
    ws = torch.empty(S.pdssm_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    sets = [dict(d=d, h=h, sel=sel, out=out)]

    def fwd(bs=None):
        bs = bs or sets[0]
        dd = bs["d"]
        S.ssm_pdssm_fwd(dd["scores"], dd["dictionary"], dd["d"], dd["bt"], h0=dd["h0"], h=bs["h"],
                        sel=bs["sel"], ws=ws, stream=stream)

    def bwd(bs=None):
        bs = bs or sets[0]
        dd = bs["d"]
        S.ssm_pdssm_bwd(dd["scores"], dd["dictionary"], dd["d"], bs["h"], bs["sel"], dd["g"], tau=1.0,
                        h0=dd["h0"], out=bs["out"], ws=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        fwd(); bwd()
    torch.cuda.synchronize()
    if S.ssm_scan_status(ws) != 0:
        raise SystemExit("device status word reports an error")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for k in range(args.steps):
        flush()
        e = ev[k]
        e[0].record(stream); fwd(); e[1].record(stream); bwd(); e[2].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    t_fwd = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_bwd = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    tt = torch.tensor([t_fwd + t_bwd, t_fwd, t_bwd], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    t_step, t_fwd, t_bwd = tt.tolist()

    sets.append(dict(d={k: torch.empty_like(v) for k, v in d.items()}, h=torch.empty_like(h),
                     sel=torch.empty_like(sel), out={k: torch.empty_like(v) for k, v in out.items()}))

    def compute(bs):
        fwd(bs); bwd(bs)

    t_e2e, h2d, d2h = e2e_pipelined(torch, dev, stream, host, sets, compute,
                                    lambda bs: dict(h=bs["h"], **bs["out"]), args.steps, world, dist)

    upd_rank = w.batch * w.seqlen * w.heads * w.nstate
    value = world * upd_rank * args.steps / t_step
    hbm, peak_kind = peaks()
    fb, bb = pdssm_algorithmic_bytes(w)
    fwd_gbs = fb / (t_fwd / args.steps) / 1e9
    bwd_gbs = bb / (t_bwd / args.steps) / 1e9
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_step / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded generator: random dictionary maps, N(0,1) scores)",
            "config": pdssm_config(args, w, world),
            "roofline": {"bound": "hbm", "kernel": "ssm_pdssm_bwd call (reverse scan + score "
                         "gradient)", "achieved": bwd_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": bwd_gbs / hbm, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": bb,
                         "traffic": measured_traffic("ssm_pdssm_bwd", "pdssm.cu", w.name)},
            "hbm_frac_fwd": fwd_gbs / hbm, "hbm_frac_bwd": bwd_gbs / hbm,
            "ms_fwd": 1e3 * t_fwd / args.steps, "ms_bwd": 1e3 * t_bwd / args.steps,
            "e2e": {"value": world * upd_rank * args.steps / t_e2e, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": E2E_OVERLAP},
            "gpu_launches": 2 * S.pdssm_kernel_launches(shape, False) * args.steps,
            "clocks": clk,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = oracle_sample_pdssm(w, inp)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference_pdssm(args, w):
    """The oracle on one batch row of the Flash PD-SSM workload per step (rank 0 only)."""
    from selective_state_space_bwd_b200 import inputs as gen
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    inp = gen.pdssm_inputs(1, w.seqlen, w.heads, w.nstate, w.ndict, seed=0)
    upd = w.seqlen * w.heads * w.nstate
    times = []
    for k in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.pdssm(inp["scores"], inp["dictionary"], inp["d"], inp["bt"], inp["h0"], inp["g"],
                     tau=1.0, threads=threads)
        if k >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = upd * len(times) / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, shapes of the workload)",
            "config": pdssm_config(args, w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"1 of {w.batch} batch rows of {w.name} per step (fwd + "
                                       f"bwd in float64 on the host cores; no L2 flush)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.memory_curve:
        return memory_curve()
    from selective_state_space_bwd_b200 import inputs as gen
    w = gen.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if isinstance(w, gen.ComplexWorkload):
        return main_complex(args, w)
    if isinstance(w, gen.PdWorkload):
        return main_pdssm(args, w)

    import torch
    import torch.distributed as dist
    from selective_state_space_bwd_b200 import build, dp, ssm_scan as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    S.lib()

    dt = torch.bfloat16 if w.io == gen.BF16 else torch.float32
    inp = gen.real_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.io, w.kind, seed=rank)
    host = {k: torch.from_numpy(v).to(dt if k not in ("A_log", "Dskip") else torch.float32)
            for k, v in inp.items()}
    host = {k: v.pin_memory() for k, v in host.items()}
    R = args.dtproj
    if R:  # delta_raw comes from the projection of a rank-R input every step
        if w.io != gen.BF16:
            raise SystemExit("--dtproj needs a bf16 workload")
        pin = gen.dtproj_inputs(w.batch, w.seqlen, w.dim, R, seed=100 + rank)
        del host["delta_raw"]
        host["u"] = torch.from_numpy(pin["u"]).to(torch.bfloat16).pin_memory()
        host["w"] = torch.from_numpy(pin["w"]).to(torch.bfloat16).pin_memory()
        host["bias"] = torch.from_numpy(pin["bias"]).pin_memory()
    d = {k: v.to(dev) for k, v in host.items()}
    if R:
        d["delta_raw"] = torch.empty_like(d["x"])
        dshape = S.dtproj_shape(w.batch * w.seqlen, w.dim, R)
        wsp = torch.empty(S.dtproj_workspace_bytes(dshape, True), dtype=torch.uint8, device=dev)
        wspf = torch.empty(S.dtproj_workspace_bytes(dshape, False), dtype=torch.uint8, device=dev)
    shape = S.real_shape(w.batch, w.seqlen, w.dim, w.dstate, w.chunk,
                         S.SSM_BF16 if w.io == gen.BF16 else S.SSM_F32, args.seg_chunks)
    nC = -(-w.seqlen // w.chunk)
    y = torch.empty_like(d["x"])
    ckpt = torch.empty((w.batch, nC, w.dim, w.dstate), dtype=torch.float32, device=dev)
    out = dict(dx=torch.empty_like(d["x"]), ddelta_raw=torch.empty_like(d["x"]),
               dA_log=torch.empty_like(d["A_log"]), dB=torch.empty_like(d["Bm"]),
               dC=torch.empty_like(d["Cm"]), dD=torch.empty_like(d["Dskip"]))
    wsf = torch.empty(S.workspace_bytes(shape, False), dtype=torch.uint8, device=dev)
    wsb = torch.empty(S.workspace_bytes(shape, True), dtype=torch.uint8, device=dev)
    gbuf = torch.empty(w.dim * w.dstate + w.dim, dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    use_ex = args.zoh or args.state or args.fused_sums
    h0 = dhL = hL = None
    if args.state:
        g = torch.Generator(device="cpu").manual_seed(1234 + rank)
        h0 = torch.randn((w.batch, w.dim, w.dstate), generator=g).to(dev)
        dhL = torch.randn((w.batch, w.dim, w.dstate), generator=g).to(dev)
    if use_ex:
        hL = torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev)
        out["dh0"] = torch.empty_like(hL)
    if R:
        out["du"] = torch.empty_like(d["u"])
        out["dw"] = torch.empty((w.dim, R), dtype=torch.float32, device=dev)
        out["dbias"] = torch.empty(w.dim, dtype=torch.float32, device=dev)
        gbuf = torch.empty(w.dim * w.dstate + w.dim + w.dim * (R + 1), dtype=torch.float32, device=dev)

    def proj_fwd(dd=None):
        dd = d if dd is None else dd
        if R:
            S.ssm_dtproj_fwd(dd["u"], dd["w"], dd["bias"], delta_raw=dd["delta_raw"], ws=wspf,
                             stream=stream)

    def proj_bwd(dd=None, oo=None):
        dd = d if dd is None else dd
        oo = out if oo is None else oo
        if R:
            S.ssm_dtproj_bwd(dd["u"], dd["w"], oo["ddelta_raw"],
                             out=dict(du=oo["du"], dw=oo["dw"], dbias=oo["dbias"]), ws=wsp,
                             stream=stream)

    def fwd():
        if use_ex:
            S.ssm_scan_fwd_ex(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"],
                              zoh=args.zoh, h0=h0, chunk=w.chunk, seg_chunks=args.seg_chunks,
                              y=y, ckpt=ckpt, hL=hL, ws=wsf, stream=stream)
        else:
            S.ssm_scan_fwd(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"],
                           chunk=w.chunk, seg_chunks=args.seg_chunks, y=y, ckpt=ckpt, ws=wsf,
                           stream=stream)

    def bwd():
        if use_ex:
            S.ssm_scan_bwd_ex(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"],
                              ckpt, d["dy"], zoh=args.zoh, h0=h0, dhL=dhL, chunk=w.chunk,
                              seg_chunks=args.seg_chunks, out=out, ws=wsb, stream=stream,
                              fused_sums=args.fused_sums)
        else:
            S.ssm_scan_bwd(d["x"], d["delta_raw"], d["A_log"], d["Bm"], d["Cm"], d["Dskip"], ckpt,
                           d["dy"], chunk=w.chunk, seg_chunks=args.seg_chunks, out=out, ws=wsb,
                           stream=stream)

    def allreduce(oo=None):
        oo = out if oo is None else oo
        if world > 1:  # one collective; the projection's gradients travel in it when present
            grads = [oo["dA_log"], oo["dD"]] + ([oo["dw"], oo["dbias"]] if R else [])
            dp.allreduce_grads(grads, buf=gbuf)

    for _ in range(max(3, args.warmup)):
        proj_fwd(); fwd(); bwd(); proj_bwd(); allreduce()
    torch.cuda.synchronize()
    if S.ssm_scan_status(wsb) != 0 or S.ssm_scan_status(wsf) != 0:
        raise SystemExit("device status word reports a non-finite state")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for k in range(args.steps):
        flush()
        e = ev[k]
        e[0].record(stream); proj_fwd(); e[1].record(stream); fwd(); e[2].record(stream)
        bwd(); e[3].record(stream); proj_bwd(); e[4].record(stream)
        allreduce(); e[5].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    t_pf = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_fwd = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_bwd = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    t_pb = sum(e[3].elapsed_time(e[4]) for e in ev) / 1e3
    t_step = sum(e[0].elapsed_time(e[5]) for e in ev) / 1e3
    tt = torch.tensor([t_step, t_fwd, t_bwd, t_pf, t_pb], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    t_step, t_fwd, t_bwd, t_pf, t_pb = tt.tolist()

    # end to end: every step's inputs come from pinned host memory and every output goes back,
    # inside the timed region (two buffer sets: one step's copies run beside the next's compute)
    sets = [dict(d=d, y=y, ckpt=ckpt, out=out)]
    sets.append(dict(d={k: torch.empty_like(v) for k, v in d.items()}, y=torch.empty_like(y),
                     ckpt=torch.empty_like(ckpt), out={k: torch.empty_like(v) for k, v in out.items()}))

    def compute(bs):
        proj_fwd(bs["d"])
        if use_ex:
            S.ssm_scan_fwd_ex(bs["d"]["x"], bs["d"]["delta_raw"], bs["d"]["A_log"], bs["d"]["Bm"],
                              bs["d"]["Cm"], bs["d"]["Dskip"], zoh=args.zoh, h0=h0, chunk=w.chunk,
                              seg_chunks=args.seg_chunks, y=bs["y"], ckpt=bs["ckpt"], hL=hL, ws=wsf,
                              stream=stream)
            S.ssm_scan_bwd_ex(bs["d"]["x"], bs["d"]["delta_raw"], bs["d"]["A_log"], bs["d"]["Bm"],
                              bs["d"]["Cm"], bs["d"]["Dskip"], bs["ckpt"], bs["d"]["dy"],
                              zoh=args.zoh, h0=h0, dhL=dhL, chunk=w.chunk,
                              seg_chunks=args.seg_chunks, out=bs["out"], ws=wsb, stream=stream,
                              fused_sums=args.fused_sums)
        else:
            S.ssm_scan_fwd(bs["d"]["x"], bs["d"]["delta_raw"], bs["d"]["A_log"], bs["d"]["Bm"],
                           bs["d"]["Cm"], bs["d"]["Dskip"], chunk=w.chunk,
                           seg_chunks=args.seg_chunks, y=bs["y"], ckpt=bs["ckpt"], ws=wsf,
                           stream=stream)
            S.ssm_scan_bwd(bs["d"]["x"], bs["d"]["delta_raw"], bs["d"]["A_log"], bs["d"]["Bm"],
                           bs["d"]["Cm"], bs["d"]["Dskip"], bs["ckpt"], bs["d"]["dy"],
                           chunk=w.chunk, seg_chunks=args.seg_chunks, out=bs["out"], ws=wsb,
                           stream=stream)
        proj_bwd(bs["d"], bs["out"])
        allreduce(bs["out"])

    t_e2e, h2d, d2h = e2e_pipelined(torch, dev, stream, host, sets, compute,
                                    lambda bs: dict(y=bs["y"], **bs["out"]), args.steps, world, dist)

    upd_rank = w.batch * w.seqlen * w.dim * w.dstate
    value = world * upd_rank * args.steps / t_step
    hbm, peak_kind = peaks()
    fb, bb = algorithmic_bytes(w)
    # the projection: forward + (du and dw in one launch for R <= 64, else two) + dw reduction
    launches = (S.kernel_launches(shape, False) + S.kernel_launches(shape, True, args.fused_sums) +
                ((3 if R <= 64 else 4) if R else 0)) * args.steps
    bwd_gbs = bb / (t_bwd / args.steps) / 1e9
    fwd_gbs = fb / (t_fwd / args.steps) / 1e9
    step_gbs = (fb + bb) / ((t_fwd + t_bwd) / args.steps) / 1e9
    alu_peak, alu_mhz = alu_peak_tops()
    if args.zoh:
        fo, bo = ZOH_FWD_OPS_PER_UPDATE * upd_rank, ZOH_BWD_OPS_PER_UPDATE * upd_rank
    else:
        fo, bo = FWD_OPS_PER_UPDATE * upd_rank, BWD_OPS_PER_UPDATE * upd_rank
    bwd_tops = bo / (t_bwd / args.steps) / 1e12

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_step / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.io == gen.BF16 else "f32",
            "data": "synthetic (seeded generator, workload value distributions)",
            "config": real_config(args, w, world),
            "roofline": {"bound": "alu", "kernel": "ssm_scan_bwd call (real_bwd_kernel + "
                         "dB/dC and parameter reductions)", "achieved": bwd_tops, "peak": alu_peak,
                         "unit": "Top/s", "frac": bwd_tops / alu_peak,
                         "peak_kind": f"derived: {SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                                      f"{alu_mhz:.0f} MHz (FMA = 1 op)",
                         "algorithmic_ops_per_launch": bo,
                         "algorithmic_bytes_per_launch": bb,
                         # records exist for the Euler path without options (and with the fused
                         # sums); zero-order hold and an initial state run other instances
                         "traffic": (None if args.zoh or args.state else
                                     measured_traffic("ssm_scan_bwd (SSM_FUSED_SUMS)" if args.fused_sums
                                                      else "ssm_scan_bwd", "real_bwd.cu", w.name)),
                         **clock_roofs(clk, bwd_tops, upd_rank / (t_bwd / args.steps),
                                       BWD_EXP2_PER_UPDATE)},
            "hbm": {"achieved_bwd": bwd_gbs, "achieved_fwd": fwd_gbs, "achieved_step": step_gbs,
                    "peak": hbm, "unit": "GB/s", "peak_kind": peak_kind},
            "hbm_frac_bwd": bwd_gbs / hbm,
            "hbm_frac_fwd": fwd_gbs / hbm, "hbm_frac_step": step_gbs / hbm,
            "alu_frac_fwd": fo / (t_fwd / args.steps) / 1e12 / alu_peak,
            "ms_fwd": 1e3 * t_fwd / args.steps, "ms_bwd": 1e3 * t_bwd / args.steps,
            "e2e": {"value": world * upd_rank * args.steps / t_e2e, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": E2E_OVERLAP},
            "gpu_launches": launches,
            "clocks": clk,
        }
        if R:
            pfb, pbb, pfl = dtproj_algorithmic(w, R)
            line["dtproj"] = {
                "rank": R, "ms_fwd": 1e3 * t_pf / args.steps, "ms_bwd": 1e3 * t_pb / args.steps,
                "algorithmic_bytes_fwd": pfb, "algorithmic_bytes_bwd": pbb, "flop_per_gemm": pfl,
                "hbm_frac_fwd": pfb / (t_pf / args.steps) / 1e9 / hbm,
                "hbm_frac_bwd": pbb / (t_pb / args.steps) / 1e9 / hbm,
                "tensor_tflops_fwd": pfl / (t_pf / args.steps) / 1e12,
                "tensor_tflops_bwd": 2 * pfl / (t_pb / args.steps) / 1e12,
                "note": "bf16 tcgen05 GEMMs (TMA operands, TMEM accumulators); ms_per_step and value include both projections"}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = oracle_sample(w, inp, zoh=args.zoh)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
