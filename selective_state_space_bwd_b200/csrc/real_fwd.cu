// Real-mode forward scan with chunk-end checkpoints.
//
// Recurrence (selective SSM, "选择性状态空间模型(S3M)原理与工程实践" §1.1, Euler input term):
//   h_t = exp(delta_t A) h_{t-1} + delta_t B_t x_t,   y_t = C_t . h_t + D x_t,
//   delta = softplus(delta_raw), A = -exp(A_log).
// Only the state at the last step of every chunk of T steps is written (the checkpoints the
// backward recomputes from; "Breaking the Memory Wall ... Tiled Operator-Space Evolution",
// abstract).
//
// Work decomposition.  Thread = (channel, S consecutive states), state pairs in packed fp32x2
// arithmetic, NG = N / S adjacent lanes per channel, 32 channels per CTA; S = 4, or S = 2 when the
// grid is too small to fill the SMs.  Each CTA streams its
// time segment through shared memory in 32-step sub-tiles: while sub-tile j is processed, the
// raw inputs of sub-tile j+1 arrive by asynchronous copies (two-stage ring), so no warp waits on
// global memory.  Per sub-tile: softplus once per (t, d) into a (delta, delta*x) tile, B and C to
// fp32, then the sequential scan in groups of 8 steps; the per-channel sums of y over the NG
// lanes are a reduce-scatter, and y leaves through a staged tile with 16-byte stores.
// When the grid has too few CTAs, time is split into segments whose entering states come from a
// summary + carry pass (the local-scan / carry / correction structure of the three-phase scan in
// "Flash PD-SSM", technical summary, hardware-aware implementation).
#include "real_common.cuh"

namespace ssm {
namespace real {
namespace {

// S states per thread: 4 (two packed pairs), or 2 (one pair) for grids too small to fill the SMs,
// which doubles the warps per SM; the y group of U steps is reduce-scattered over the NG lanes.
template <int N, int S_>
struct FwdCfg {
    static constexpr int S = S_;          // states per thread
    static constexpr int P2 = S / 2;      // state pairs per thread
    static constexpr int NG = N / S;      // lanes per channel
    static constexpr int DT = kRealDT;    // channels per CTA
    static constexpr int NT = DT * NG;    // threads per CTA
    static constexpr int TT = 32;         // steps per staged sub-tile
    static constexpr int U = 8;           // steps per unrolled group (>= NG)
    static_assert(U >= NG, "one y value per lane at least");
};

template <typename E, int N>
struct FwdSmem {
    static constexpr int TT = FwdCfg<N, 4>::TT, DT = FwdCfg<N, 4>::DT;
    static constexpr int XE = TT * DT;                                  // elements of an x tile
    static constexpr int BE = TT * N;                                   // elements of a B tile
    static constexpr int STAGE = (2 * XE + 2 * BE) * (int)sizeof(E);    // x, delta_raw, B, C
    static constexpr int DD = 2 * STAGE;                                // (delta, delta*x) float2
    static constexpr int BF = DD + XE * 8;                              // B as fp32
    static constexpr int CF = BF + BE * 4;                              // C as fp32
    static constexpr int Y = CF + BE * 4;                               // y tile
    static constexpr int BYTES = Y + XE * (int)sizeof(E);
};

// SUMMARY = true: local scan from zero over segments 0..nseg-2, emitting (prod a, end state).
// SUMMARY = false: the scan from the segment's entering state, writing y and checkpoints.
template <typename E, int N, int S, bool SUMMARY, bool ZOH>
__global__ void __launch_bounds__(FwdCfg<N, S>::NT) real_fwd_kernel(RealArgs p) {
    using Cfg = FwdCfg<N, S>;
    using Sm = FwdSmem<E, N>;
    constexpr int P2 = Cfg::P2, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT, TT = Cfg::TT;
    constexpr int U = SUMMARY ? 16 : Cfg::U;  // the segment summaries (no y) scan 16-step groups
    extern __shared__ __align__(16) unsigned char smem[];
    float2* sdd = reinterpret_cast<float2*>(smem + Sm::DD);
    float* sBf = reinterpret_cast<float*>(smem + Sm::BF);
    float* sCf = reinterpret_cast<float*>(smem + Sm::CF);
    E* sy = reinterpret_cast<E*>(smem + Sm::Y);

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * Cfg::S;
    const bool dv = d < p.D;
    const int T = p.T;
    const int TTe = T < TT ? T : TT;     // sub-tile length (a sub-tile never crosses a chunk end)
    const int t_begin = seg * p.seg_chunks * T;
    const int t_end = min(p.L, min(p.nC, (seg + 1) * p.seg_chunks) * T);
    const int ntiles = (t_end - t_begin + TTe - 1) / TTe;

    float2 A2[P2], h[P2], P[P2];
    float2 Ar[P2];  // zero-order hold: 1 / A
#pragma unroll
    for (int i = 0; i < P2; ++i) {
        A2[i] = dv ? make_float2(-expf(p.A_log[d * N + n0 + 2 * i]) * kLog2e,
                                 -expf(p.A_log[d * N + n0 + 2 * i + 1]) * kLog2e)
                   : make_float2(0.0f, 0.0f);
        if (ZOH)
            Ar[i] = dv ? make_float2(-expf(-p.A_log[d * N + n0 + 2 * i]),
                                     -expf(-p.A_log[d * N + n0 + 2 * i + 1]))
                       : make_float2(0.0f, 0.0f);
        h[i] = make_float2(0.0f, 0.0f);
        P[i] = make_float2(1.0f, 1.0f);
    }
    if (!SUMMARY && dv) {
        // the state entering this segment: from the carry when split in time, else h0 (or zero)
        const float* src = p.nseg > 1 ? p.hin + (((size_t)b * p.nseg + seg) * p.D + d) * N + n0
                           : p.h0   ? p.h0 + ((size_t)b * p.D + d) * N + n0
                                    : nullptr;
        if (src) ld_pairs<S>(h, src);
    }
    const size_t boff = (size_t)b * p.L;
    const E* xb = static_cast<const E*>(p.x) + boff * p.D;
    const E* drb = static_cast<const E*>(p.draw) + boff * p.D;
    const E* Bb = static_cast<const E*>(p.Bm) + boff * N;
    const E* Cb = static_cast<const E*>(p.Cm) + boff * N;
    E* yb = SUMMARY ? nullptr : static_cast<E*>(p.y) + boff * p.D;
    const float dsk = (!SUMMARY && dv) ? p.Dskip[d] : 0.0f;

    auto stage_x = [&](int k) { return reinterpret_cast<E*>(smem + k * Sm::STAGE); };
    auto issue = [&](int j, int k) {
        const int t0 = t_begin + j * TTe;
        const int rows4 = (min(TTe, p.L - t0) + U - 1) / U * U;
        E* sx = stage_x(k);
        cp_async_tile<E, DT>(sx, xb, t0, rows4, p.L, d0, p.D, tid, NT);
        cp_async_tile<E, DT>(sx + Sm::XE, drb, t0, rows4, p.L, d0, p.D, tid, NT);
        cp_async_flat<E>(sx + 2 * Sm::XE, Bb, (size_t)t0 * N, rows4 * N, (size_t)p.L * N, tid, NT);
        if (!SUMMARY)
            cp_async_flat<E>(sx + 2 * Sm::XE + Sm::BE, Cb, (size_t)t0 * N, rows4 * N,
                             (size_t)p.L * N, tid, NT);
        cp_async_commit();
    };

    // input term w B_t x_t for a pair of states given (delta, delta x), a = exp(delta A) and
    // zl2 = delta A log2(e): w = delta (Euler) or (exp(delta A) - 1) / A (zero-order hold)
    auto input_term = [&](float2 dd, float2 a, float2 zl2, float2 bq, int i) {
        if constexpr (ZOH) {
            const float2 z = __fmul2_rn(zl2, f2(kLn2));
            const float2 rz = __fmul2_rn(f2(__fdividef(1.0f, dd.x)), Ar[i]);
            return __fmul2_rn(__fmul2_rn(f2(dd.y), zoh_e1(z, a, rz)), bq);
        } else {
            return __fmul2_rn(f2(dd.y), bq);
        }
    };

    if (ntiles > 0) issue(0, 0);
    for (int j = 0; j < ntiles; ++j) {
        const int k = j & 1;
        if (j + 1 < ntiles) {
            issue(j + 1, k ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int t0 = t_begin + j * TTe;
        const int rows = min(TTe, p.L - t0);
        const int rows4 = (rows + U - 1) / U * U;
        const E* sx = stage_x(k);
        const E* sdr = sx + Sm::XE;
        const E* sB = sx + 2 * Sm::XE;
        const E* sC = sB + Sm::BE;
        // steps past the sequence end get delta = 0: a = 1 and no input, i.e. they change nothing
        for (int i = tid; i < rows4 * DT; i += NT) {
            const float dlt = i < rows * DT ? softplus_fast(Elem<E>::to_f(sdr[i])) : 0.0f;
            sdd[i] = make_float2(dlt, dlt * Elem<E>::to_f(sx[i]));
        }
        for (int i = tid; i < rows4 * N; i += NT) {
            sBf[i] = Elem<E>::to_f(sB[i]);
            if (!SUMMARY) sCf[i] = Elem<E>::to_f(sC[i]);
        }
        __syncthreads();
        for (int r0 = 0; r0 < rows; r0 += U) {
            float yp[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u;
                const float2 dd = sdd[r * DT + dl];
                float2 bq[P2];
                ld_pairs<S>(bq, sBf + r * N + n0);
                if (SUMMARY) {
#pragma unroll
                    for (int i = 0; i < P2; ++i) {
                        const float2 zl2 = __fmul2_rn(f2(dd.x), A2[i]);
                        const float2 a = ex2_pair(zl2);
                        h[i] = __ffma2_rn(a, h[i], input_term(dd, a, zl2, bq[i], i));
                        P[i] = __fmul2_rn(P[i], a);
                    }
                } else {
                    float2 cq[P2];
                    ld_pairs<S>(cq, sCf + r * N + n0);
                    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int i = 0; i < P2; ++i) {
                        const float2 zl2 = __fmul2_rn(f2(dd.x), A2[i]);
                        const float2 a = ex2_pair(zl2);
                        h[i] = __ffma2_rn(a, h[i], input_term(dd, a, zl2, bq[i], i));
                        acc = __ffma2_rn(cq[i], h[i], acc);
                    }
                    yp[u] = acc.x + acc.y;
                }
            }
            if (!SUMMARY) {
                reduce_scatter<U, NG>(yp, ng);
#pragma unroll
                for (int jj = 0; jj < U / NG; ++jj) {
                    const int r = r0 + ng * (U / NG) + jj;
                    if (r < rows)
                        sy[r * DT + dl] = Elem<E>::from_f(fmaf(dsk, Elem<E>::to_f(sx[r * DT + dl]), yp[jj]));
                }
            }
        }
        const bool chunk_end = (t0 + rows) % T == 0 || t0 + rows == p.L;
        if (!SUMMARY && dv && chunk_end) {
            st_pairs<S>(p.ckpt + (((size_t)b * p.nC + t0 / T) * p.D + d) * N + n0, h);
            if (p.hL && t0 + rows == p.L) st_pairs<S>(p.hL + ((size_t)b * p.D + d) * N + n0, h);
        }
        __syncthreads();
        if (!SUMMARY) store_tile<E, DT>(yb, sy, t0, rows, p.L, d0, p.D, tid, NT);
    }
    if (SUMMARY) {
        if (dv) {
            const size_t o = (((size_t)b * (p.nseg - 1) + seg) * p.D + d) * N + n0;
            st_pairs<S>(p.sumP + o, P);
            st_pairs<S>(p.sumS + o, h);
        }
    } else if (dv && !all_finite<S>(h)) {
        flag_status(p.status, kStatusNonFinite);
    }
}

// State entering each segment: h_in[0] = h0 (or 0), h_in[s+1] = P_s h_in[s] + S_s.
__global__ void real_carry_fwd_kernel(int B, int nseg, int DN, const float* __restrict__ P,
                                      const float* __restrict__ Sv, float* __restrict__ hin,
                                      const float* __restrict__ h0) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * DN) return;
    const int b = (int)(i / DN), k = (int)(i % DN);
    float h = h0 ? h0[i] : 0.0f;
    for (int s = 0; s < nseg; ++s) {
        hin[((size_t)b * nseg + s) * DN + k] = h;
        if (s < nseg - 1) {
            const size_t j = ((size_t)b * (nseg - 1) + s) * DN + k;
            h = fmaf(P[j], h, Sv[j]);
        }
    }
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename E, int N, int S, bool ZOH>
cudaError_t real_fwd_impl(const RealArgs& a, cudaStream_t st) {
    const dim3 block(FwdCfg<N, S>::NT);
    const size_t sm = FwdSmem<E, N>::BYTES;
    cudaError_t e;
    if (a.nseg > 1) {
        if ((e = set_smem(real_fwd_kernel<E, N, S, true, ZOH>, sm)) != cudaSuccess) return e;
        real_fwd_kernel<E, N, S, true, ZOH><<<dim3(a.ndt, a.B, a.nseg - 1), block, sm, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.D * N;
        real_carry_fwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.B, a.nseg, a.D * N,
                                                                            a.sumP, a.sumS, a.hin,
                                                                            a.h0);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = set_smem(real_fwd_kernel<E, N, S, false, ZOH>, sm)) != cudaSuccess) return e;
    real_fwd_kernel<E, N, S, false, ZOH><<<dim3(a.ndt, a.B, a.nseg), block, sm, st>>>(a);
    return cudaGetLastError();
}

// Two states per thread when the main launch has fewer CTAs than 3 per SM on 148 SMs (444): the
// grid then gives under 12 warps per SM at four states per thread, too few to hide the latency
// of the exp / FMA chain; above that the extra per-step work of the narrower threads costs more
// than the latency it hides.
constexpr int64_t kFwdNarrowCtas = 444;

template <typename E, int N, bool ZOH>
cudaError_t real_fwd_pick(const RealArgs& a, cudaStream_t st) {
    if ((int64_t)a.ndt * a.B * a.nseg < kFwdNarrowCtas) return real_fwd_impl<E, N, 2, ZOH>(a, st);
    return real_fwd_impl<E, N, 4, ZOH>(a, st);
}

template <typename E, bool ZOH>
cudaError_t fwd_dispatch_n(const RealArgs& a, int N, cudaStream_t st) {
    if (N == 4) return real_fwd_pick<E, 4, ZOH>(a, st);
    if (N == 8) return real_fwd_pick<E, 8, ZOH>(a, st);
    return real_fwd_pick<E, 16, ZOH>(a, st);
}

template <typename E>
cudaError_t fwd_dispatch(const RealArgs& a, int N, cudaStream_t st) {
    return a.zoh ? fwd_dispatch_n<E, true>(a, N, st) : fwd_dispatch_n<E, false>(a, N, st);
}

}  // namespace
}  // namespace real

cudaError_t launch_real_fwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st) {
    return io_bf16 ? real::fwd_dispatch<__nv_bfloat16>(a, N, st) : real::fwd_dispatch<float>(a, N, st);
}

}  // namespace ssm
