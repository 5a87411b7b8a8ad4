// Real-mode selective scan: forward with chunk checkpoints, exact chunk-recomputing backward.
//
// Recurrence (selective SSM, "选择性状态空间模型(S3M)原理与工程实践" §1.1, Euler input term):
//   h_t = exp(delta_t A) h_{t-1} + delta_t B_t x_t,   y_t = C_t . h_t + D x_t,
//   delta = softplus(delta_raw), A = -exp(A_log).
// Backward ("Breaking the Memory Wall ... Tiled Operator-Space Evolution", abstract): only the
// state at every chunk end is kept; each chunk is recomputed from its checkpoint and the exact
// adjoint g_t = C_t dy_t + a_{t+1} g_{t+1} is swept backwards through it.
//
// Work decomposition.  Thread = (channel d, S consecutive states).  A CTA owns DT channels of one
// batch row and one time segment (a run of whole chunks).  When a segment does not start at t=0
// its entering state comes from a carry pass over per-segment summaries (prod a, local end state)
// — the local-scan / carry / correction structure of the three-phase scan in "Flash PD-SSM"
// (technical summary, hardware-aware implementation).  The backward mirrors it in reverse time.
#include "ssm_device.cuh"
#include "ssm_internal.h"

namespace ssm {
namespace {

template <int N>
struct RealCfg {
    static constexpr int S = kRealS;
    static constexpr int NG = N / S;
    static constexpr int DT = kRealDT;
    static constexpr int NT = DT * NG;
    static constexpr int TS = kRealTS;
    static_assert(N % S == 0 && NG >= 1 && NG <= 4, "dstate must be 4, 8 or 16");
};

__device__ __forceinline__ bool all_finite4(const float* v) {
    return isfinite(v[0]) && isfinite(v[1]) && isfinite(v[2]) && isfinite(v[3]);
}

// ------------------------------------------------------------------------------------------------
// Forward.  SUMMARY = true: local scan from zero over segments 0..nseg-2, emitting (prod a, end
// state).  SUMMARY = false: the real scan from the segment's entering state, writing y and the
// chunk-end checkpoints.
// Shared memory: x, delta_raw raw tiles [T][DT] (delta_raw's is reused for y), B, C as float
// [T][N], (delta, delta*x) pairs [T][DT].
template <typename E, int N, bool SUMMARY>
__global__ void __launch_bounds__(RealCfg<N>::NT) real_fwd_kernel(RealArgs p) {
    using Cfg = RealCfg<N>;
    constexpr int S = Cfg::S, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT;
    extern __shared__ __align__(16) unsigned char smem[];
    const int T = p.T;
    E* sx = reinterpret_cast<E*>(smem);
    E* sdr = sx + T * DT;
    float* sB = reinterpret_cast<float*>(sdr + T * DT);
    float* sC = sB + T * N;
    float2* sdd = reinterpret_cast<float2*>(sC + T * N);

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * S;
    const bool dv = d < p.D;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);

    float A2[S], h[S], P[S];
#pragma unroll
    for (int j = 0; j < S; ++j) {
        A2[j] = dv ? -expf(p.A_log[d * N + n0 + j]) * kLog2e : 0.0f;
        h[j] = 0.0f;
        P[j] = 1.0f;
    }
    if (!SUMMARY && seg > 0 && dv) {
        const float4 hv = *reinterpret_cast<const float4*>(
            p.hin + (((size_t)b * p.nseg + seg) * p.D + d) * N + n0);
        h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
    }
    const size_t boff = (size_t)b * p.L;
    const E* xb = static_cast<const E*>(p.x) + boff * p.D;
    const E* drb = static_cast<const E*>(p.draw) + boff * p.D;
    const E* Bb = static_cast<const E*>(p.Bm) + boff * N;
    const E* Cb = static_cast<const E*>(p.Cm) + boff * N;
    E* yb = SUMMARY ? nullptr : static_cast<E*>(p.y) + boff * p.D;
    const float dsk = (!SUMMARY && dv) ? p.Dskip[d] : 0.0f;

    for (int c = c_begin; c < c_end; ++c) {
        const int t0 = c * T;
        const int rows = min(T, p.L - t0);
        __syncthreads();
        load_tile<E, DT>(sx, xb, t0, rows, p.L, d0, p.D, tid, NT);
        load_tile<E, DT>(sdr, drb, t0, rows, p.L, d0, p.D, tid, NT);
        load_rows_f32<E, N>(sB, Bb, t0, rows, p.L, tid, NT);
        if (!SUMMARY) load_rows_f32<E, N>(sC, Cb, t0, rows, p.L, tid, NT);
        __syncthreads();
        for (int i = tid; i < rows * DT; i += NT) {
            const float dlt = softplus_acc(Elem<E>::to_f(sdr[i]));
            sdd[i] = make_float2(dlt, dlt * Elem<E>::to_f(sx[i]));
        }
        __syncthreads();
        for (int r = 0; r < rows; ++r) {
            const float2 dd = sdd[r * DT + dl];
            const float4 bv = *reinterpret_cast<const float4*>(sB + r * N + n0);
            const float bj[4] = {bv.x, bv.y, bv.z, bv.w};
            if (SUMMARY) {
#pragma unroll
                for (int j = 0; j < S; ++j) {
                    const float a = ex2_mufu(dd.x * A2[j]);
                    h[j] = fmaf(a, h[j], dd.y * bj[j]);
                    P[j] *= a;
                }
            } else {
                const float4 cv = *reinterpret_cast<const float4*>(sC + r * N + n0);
                const float cj[4] = {cv.x, cv.y, cv.z, cv.w};
                float yp = 0.0f;
#pragma unroll
                for (int j = 0; j < S; ++j) {
                    const float a = ex2_mufu(dd.x * A2[j]);
                    h[j] = fmaf(a, h[j], dd.y * bj[j]);
                    yp = fmaf(cj[j], h[j], yp);
                }
#pragma unroll
                for (int o = 1; o < NG; o <<= 1) yp += __shfl_xor_sync(0xffffffffu, yp, o);
                if (ng == 0)
                    sdr[r * DT + dl] = Elem<E>::from_f(fmaf(dsk, Elem<E>::to_f(sx[r * DT + dl]), yp));
            }
        }
        if (!SUMMARY) {
            if (dv)
                *reinterpret_cast<float4*>(p.ckpt + (((size_t)b * p.nC + c) * p.D + d) * N + n0) =
                    make_float4(h[0], h[1], h[2], h[3]);
            __syncthreads();
            store_tile<E, DT>(yb, sdr, t0, rows, p.L, d0, p.D, tid, NT);
        }
    }
    if (SUMMARY) {
        if (dv) {
            const size_t o = (((size_t)b * (p.nseg - 1) + seg) * p.D + d) * N + n0;
            *reinterpret_cast<float4*>(p.sumP + o) = make_float4(P[0], P[1], P[2], P[3]);
            *reinterpret_cast<float4*>(p.sumS + o) = make_float4(h[0], h[1], h[2], h[3]);
        }
    } else if (dv && !all_finite4(h)) {
        flag_status(p.status, kStatusNonFinite);
    }
}

// State entering each segment: h_in[0] = 0, h_in[s+1] = P_s h_in[s] + S_s.
__global__ void real_carry_fwd_kernel(int B, int nseg, int DN, const float* __restrict__ P,
                                      const float* __restrict__ Sv, float* __restrict__ hin) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * DN) return;
    const int b = (int)(i / DN), k = (int)(i % DN);
    float h = 0.0f;
    for (int s = 0; s < nseg; ++s) {
        hin[((size_t)b * nseg + s) * DN + k] = h;
        if (s < nseg - 1) {
            const size_t j = ((size_t)b * (nseg - 1) + s) * DN + k;
            h = fmaf(P[j], h, Sv[j]);
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Backward segment summary (segments 1..nseg-1): local reverse adjoint from zero over the
// segment, v <- a_t (C_t dy_t + v), and P = prod a over the segment.
template <typename E, int N>
__global__ void __launch_bounds__(RealCfg<N>::NT) real_bwd_summary_kernel(RealArgs p) {
    using Cfg = RealCfg<N>;
    constexpr int S = Cfg::S, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT;
    extern __shared__ __align__(16) unsigned char smem[];
    const int T = p.T;
    E* sdy = reinterpret_cast<E*>(smem);
    E* sdr = sdy + T * DT;
    float* sC = reinterpret_cast<float*>(sdr + T * DT);
    float* sdel = sC + T * N;

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int b = blockIdx.y, seg = blockIdx.z + 1;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * S;
    const bool dv = d < p.D;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);

    float A2[S], v[S], P[S];
#pragma unroll
    for (int j = 0; j < S; ++j) {
        A2[j] = dv ? -expf(p.A_log[d * N + n0 + j]) * kLog2e : 0.0f;
        v[j] = 0.0f;
        P[j] = 1.0f;
    }
    const size_t boff = (size_t)b * p.L;
    const E* dyb = static_cast<const E*>(p.dy) + boff * p.D;
    const E* drb = static_cast<const E*>(p.draw) + boff * p.D;
    const E* Cb = static_cast<const E*>(p.Cm) + boff * N;

    for (int c = c_end - 1; c >= c_begin; --c) {
        const int t0 = c * T;
        const int rows = min(T, p.L - t0);
        __syncthreads();
        load_tile<E, DT>(sdy, dyb, t0, rows, p.L, d0, p.D, tid, NT);
        load_tile<E, DT>(sdr, drb, t0, rows, p.L, d0, p.D, tid, NT);
        load_rows_f32<E, N>(sC, Cb, t0, rows, p.L, tid, NT);
        __syncthreads();
        for (int i = tid; i < rows * DT; i += NT) sdel[i] = softplus_acc(Elem<E>::to_f(sdr[i]));
        __syncthreads();
        for (int r = rows - 1; r >= 0; --r) {
            const float dlt = sdel[r * DT + dl];
            const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
            const float4 cv = *reinterpret_cast<const float4*>(sC + r * N + n0);
            const float cj[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int j = 0; j < S; ++j) {
                const float a = ex2_mufu(dlt * A2[j]);
                v[j] = a * fmaf(cj[j], dyv, v[j]);
                P[j] *= a;
            }
        }
    }
    if (dv) {
        const size_t o = (((size_t)b * (p.nseg - 1) + (seg - 1)) * p.D + d) * N + n0;
        *reinterpret_cast<float4*>(p.gsumP + o) = make_float4(P[0], P[1], P[2], P[3]);
        *reinterpret_cast<float4*>(p.gsumG + o) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// Scaled adjoint entering each segment from its end: v_in[nseg-1] = 0,
// v_in[s-1] = G_s + P_s v_in[s].
__global__ void real_carry_bwd_kernel(int B, int nseg, int DN, const float* __restrict__ P,
                                      const float* __restrict__ G, float* __restrict__ vin) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * DN) return;
    const int b = (int)(i / DN), k = (int)(i % DN);
    float v = 0.0f;
    for (int s = nseg - 1; s >= 0; --s) {
        vin[((size_t)b * nseg + s) * DN + k] = v;
        if (s > 0) {
            const size_t j = ((size_t)b * (nseg - 1) + (s - 1)) * DN + k;
            v = fmaf(P[j], v, G[j]);
        }
    }
}

// Reduce 8 per-lane values over the lanes that share (lane % NG).  On return v[0] holds the total
// of value index ((lane>>4)&1)*4 + ((lane>>3)&1)*2 + ((lane>>2)&1).
template <int NG>
__device__ __forceinline__ void transpose_reduce8(float (&v)[8]) {
    const int lane = threadIdx.x & 31;
    {
        const bool up = lane & 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = up ? v[i] : v[i + 4];
            const float keep = up ? v[i + 4] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
    }
    {
        const bool up = lane & 8;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = up ? v[i] : v[i + 2];
            const float keep = up ? v[i + 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    {
        const bool up = lane & 4;
        const float send = up ? v[0] : v[1];
        const float keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    if (NG <= 2) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    if (NG <= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// ------------------------------------------------------------------------------------------------
// Backward main kernel.  For every stretch of TB <= 128 steps (a chunk, or half a 256-step
// chunk), in reverse order:
//   pass A: recompute h forward from the chunk checkpoint, saving h every TS steps (smem);
//   pass B: for each TS-step piece in reverse, recompute (a_t, a_t h_{t-1}) into registers and
//           sweep the adjoint backwards, emitting dx, ddelta_raw (per channel), per-CTA sums of
//           dB, dC (over the CTA's channels) and per-thread sums for dA_log, dD.
// Shared memory: x, delta_raw, dy raw tiles [TB][DT]; B, C float [TB][N]; delta [TB][DT];
// saved states [TB/TS][NT] float4; cross-warp dB/dC sums [TS][warps][2N].
template <typename E, int N>
__global__ void __launch_bounds__(RealCfg<N>::NT) real_bwd_kernel(RealArgs p) {
    using Cfg = RealCfg<N>;
    constexpr int S = Cfg::S, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT, TS = Cfg::TS;
    constexpr int NW = NT / 32, N2 = 2 * N;
    extern __shared__ __align__(16) unsigned char smem[];
    const int T = p.T;
    const int TB = min(T, kRealMaxTB);
    E* sx = reinterpret_cast<E*>(smem);
    E* sdr = sx + TB * DT;
    E* sdy = sdr + TB * DT;
    float* sB = reinterpret_cast<float*>(sdy + TB * DT);
    float* sC = sB + TB * N;
    float* sdel = sC + TB * N;
    float4* sbnd = reinterpret_cast<float4*>(sdel + TB * DT);
    float* sred = reinterpret_cast<float*>(sbnd + (TB / TS) * NT);

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * S;
    const bool dv = d < p.D;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);
    // which of the 2N (dB, dC) sums this lane carries after transpose_reduce8, and whether it
    // is the lane that writes it
    const int ridx = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
    const int rout = ridx < S ? n0 + ridx : N + n0 + (ridx - S);
    const bool rwriter = (NG == 4) || (NG == 2 && !(lane & 2)) || (NG == 1 && !(lane & 3));

    float A[S], A2[S], v[S], dA[S];
#pragma unroll
    for (int j = 0; j < S; ++j) {
        A[j] = dv ? -expf(p.A_log[d * N + n0 + j]) : 0.0f;
        A2[j] = A[j] * kLog2e;
        v[j] = 0.0f;
        dA[j] = 0.0f;
    }
    if (seg < p.nseg - 1 && dv) {
        const float4 vv = *reinterpret_cast<const float4*>(
            p.vin + (((size_t)b * p.nseg + seg) * p.D + d) * N + n0);
        v[0] = vv.x; v[1] = vv.y; v[2] = vv.z; v[3] = vv.w;
    }
    float dDacc = 0.0f;
    const float dsk = dv ? p.Dskip[d] : 0.0f;
    const size_t boff = (size_t)b * p.L;
    const E* xb = static_cast<const E*>(p.x) + boff * p.D;
    const E* drb = static_cast<const E*>(p.draw) + boff * p.D;
    const E* dyb = static_cast<const E*>(p.dy) + boff * p.D;
    const E* Bb = static_cast<const E*>(p.Bm) + boff * N;
    const E* Cb = static_cast<const E*>(p.Cm) + boff * N;
    E* dxb = static_cast<E*>(p.dx) + boff * p.D;
    E* ddrb = static_cast<E*>(p.ddraw) + boff * p.D;
    float* partb = p.dBC_part + ((size_t)blockIdx.x * p.B + b) * (size_t)p.L * N2;

    const int per_chunk = T / TB;  // 1, or 2 for 256-step chunks
    for (int c = c_end - 1; c >= c_begin; --c) {
        for (int part = per_chunk - 1; part >= 0; --part) {
            const int t0 = c * T + part * TB;
            if (t0 >= p.L) continue;
            const int rows = min(TB, p.L - t0);
            // state entering this stretch
            float h[S];
            if (c > 0 && dv) {
                const float4 hv = *reinterpret_cast<const float4*>(
                    p.ckpt_in + (((size_t)b * p.nC + (c - 1)) * p.D + d) * N + n0);
                h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
            } else {
#pragma unroll
                for (int j = 0; j < S; ++j) h[j] = 0.0f;
            }
            for (int pre = 0; pre < part; ++pre) {  // advance through earlier stretches of the chunk
                const int tp = c * T + pre * TB;
                __syncthreads();
                load_tile<E, DT>(sx, xb, tp, TB, p.L, d0, p.D, tid, NT);
                load_tile<E, DT>(sdr, drb, tp, TB, p.L, d0, p.D, tid, NT);
                load_rows_f32<E, N>(sB, Bb, tp, TB, p.L, tid, NT);
                __syncthreads();
                for (int r = 0; r < TB; ++r) {
                    const float dlt = softplus_acc(Elem<E>::to_f(sdr[r * DT + dl]));
                    const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                    const float4 bv = *reinterpret_cast<const float4*>(sB + r * N + n0);
                    const float bj[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int j = 0; j < S; ++j) h[j] = fmaf(ex2_mufu(dlt * A2[j]), h[j], dxv * bj[j]);
                }
            }
            __syncthreads();
            load_tile<E, DT>(sx, xb, t0, rows, p.L, d0, p.D, tid, NT);
            load_tile<E, DT>(sdr, drb, t0, rows, p.L, d0, p.D, tid, NT);
            load_tile<E, DT>(sdy, dyb, t0, rows, p.L, d0, p.D, tid, NT);
            load_rows_f32<E, N>(sB, Bb, t0, rows, p.L, tid, NT);
            load_rows_f32<E, N>(sC, Cb, t0, rows, p.L, tid, NT);
            __syncthreads();
            for (int i = tid; i < rows * DT; i += NT) sdel[i] = softplus_acc(Elem<E>::to_f(sdr[i]));
            __syncthreads();

            // pass A: forward recompute, saving the state at the start of every TS-step piece
            const int npieces = (rows + TS - 1) / TS;
            for (int k = 0; k < npieces; ++k) {
                sbnd[k * NT + tid] = make_float4(h[0], h[1], h[2], h[3]);
                const int r1 = min(rows, (k + 1) * TS);
                for (int r = k * TS; r < r1; ++r) {
                    const float dlt = sdel[r * DT + dl];
                    const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                    const float4 bv = *reinterpret_cast<const float4*>(sB + r * N + n0);
                    const float bj[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int j = 0; j < S; ++j) h[j] = fmaf(ex2_mufu(dlt * A2[j]), h[j], dxv * bj[j]);
                }
            }

            // pass B: pieces in reverse
            for (int k = npieces - 1; k >= 0; --k) {
                const int r0 = k * TS;
                const int nr = min(TS, rows - r0);
                float aa[TS][S], pp[TS][S];
                {
                    const float4 hv = sbnd[k * NT + tid];
                    float hc[S] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                    for (int ts = 0; ts < TS; ++ts) {
                        if (ts < nr) {
                            const int r = r0 + ts;
                            const float dlt = sdel[r * DT + dl];
                            const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                            const float4 bv = *reinterpret_cast<const float4*>(sB + r * N + n0);
                            const float bj[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                            for (int j = 0; j < S; ++j) {
                                const float a = ex2_mufu(dlt * A2[j]);
                                const float pr = a * hc[j];
                                aa[ts][j] = a;
                                pp[ts][j] = pr;
                                hc[j] = fmaf(dxv, bj[j], pr);
                            }
                        }
                    }
                }
#pragma unroll
                for (int ts = TS - 1; ts >= 0; --ts) {
                    if (ts < nr) {
                        const int r = r0 + ts;
                        const float dlt = sdel[r * DT + dl];
                        const float xv = Elem<E>::to_f(sx[r * DT + dl]);
                        const float dxv = dlt * xv;
                        const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                        const float4 bv = *reinterpret_cast<const float4*>(sB + r * N + n0);
                        const float4 cv = *reinterpret_cast<const float4*>(sC + r * N + n0);
                        const float bj[4] = {bv.x, bv.y, bv.z, bv.w};
                        const float cj[4] = {cv.x, cv.y, cv.z, cv.w};
                        float sgB = 0.0f, sAq = 0.0f;
                        float red[8];
#pragma unroll
                        for (int j = 0; j < S; ++j) {
                            const float g = fmaf(cj[j], dyv, v[j]);
                            const float hj = fmaf(dxv, bj[j], pp[ts][j]);
                            const float q = g * pp[ts][j];
                            dA[j] = fmaf(dlt, q, dA[j]);
                            sAq = fmaf(A[j], q, sAq);
                            sgB = fmaf(g, bj[j], sgB);
                            red[j] = g * dxv;
                            red[S + j] = dyv * hj;
                            v[j] = aa[ts][j] * g;
                        }
#pragma unroll
                        for (int o = 1; o < NG; o <<= 1) {
                            sgB += __shfl_xor_sync(0xffffffffu, sgB, o);
                            sAq += __shfl_xor_sync(0xffffffffu, sAq, o);
                        }
                        transpose_reduce8<NG>(red);
                        if (rwriter) sred[(ts * NW + warp) * N2 + rout] = red[0];
                        if (ng == 0) {
                            const float zr = Elem<E>::to_f(sdr[r * DT + dl]);
                            const float dxo = fmaf(dsk, dyv, dlt * sgB);
                            const float ddel = fmaf(xv, sgB, sAq);
                            sx[r * DT + dl] = Elem<E>::from_f(dxo);          // x no longer needed
                            sdr[r * DT + dl] = Elem<E>::from_f(ddel * sigmoid_acc(zr));
                            dDacc = fmaf(dyv, xv, dDacc);
                        }
                    }
                }
                __syncthreads();
                for (int i = tid; i < nr * N2; i += NT) {
                    const int ts = i / N2, o = i - ts * N2;
                    float s = 0.0f;
#pragma unroll
                    for (int w = 0; w < NW; ++w) s += sred[(ts * NW + w) * N2 + o];
                    partb[(size_t)(t0 + r0 + ts) * N2 + o] = s;
                }
                __syncthreads();
            }
            store_tile<E, DT>(dxb, sx, t0, rows, p.L, d0, p.D, tid, NT);
            store_tile<E, DT>(ddrb, sdr, t0, rows, p.L, d0, p.D, tid, NT);
        }
    }
    if (dv) {
        const size_t o = (((size_t)b * p.nseg + seg) * p.D + d) * N + n0;
        *reinterpret_cast<float4*>(p.dA_part + o) = make_float4(dA[0], dA[1], dA[2], dA[3]);
        if (ng == 0) p.dD_part[((size_t)b * p.nseg + seg) * p.D + d] = dDacc;
        if (!all_finite4(v)) flag_status(p.status, kStatusNonFinite);
    }
}

// dB, dC: fixed-order sums of the per-CTA partials over the channel tiles.
template <typename E, int N>
__global__ void real_reduce_dbc_kernel(RealArgs p) {
    constexpr int N2 = 2 * N;
    const int64_t total = (int64_t)p.B * p.L * N2;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total) return;
    const int64_t bl = i / N2;
    const int o = (int)(i - bl * N2);
    const size_t stride = (size_t)p.B * p.L * N2;
    float s = 0.0f;
    for (int t = 0; t < p.ndt; ++t) s += p.dBC_part[(size_t)t * stride + i];
    if (o < N)
        static_cast<E*>(p.dB)[bl * N + o] = Elem<E>::from_f(s);
    else
        static_cast<E*>(p.dC)[bl * N + (o - N)] = Elem<E>::from_f(s);
}

// dA_log = A * sum over (batch, segment) of the per-thread sums of delta*q; dD likewise.
__global__ void real_reduce_params_kernel(RealArgs p, int N) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t DN = (int64_t)p.D * N;
    const int BS = p.B * p.nseg;
    if (i < DN) {
        float s = 0.0f;
        for (int k = 0; k < BS; ++k) s += p.dA_part[(size_t)k * DN + i];
        p.dA_log[i] = -expf(p.A_log[i]) * s;
    }
    if (i < p.D) {
        float s = 0.0f;
        for (int k = 0; k < BS; ++k) s += p.dD_part[(size_t)k * p.D + i];
        p.dD[i] = s;
    }
}

size_t fwd_smem(int T, int N, int esz) {
    const int DT = kRealDT;
    return (size_t)T * DT * esz * 2 + (size_t)T * N * 4 * 2 + (size_t)T * DT * 8;
}
size_t bwd_summary_smem(int T, int N, int esz) {
    const int DT = kRealDT;
    return (size_t)T * DT * esz * 2 + (size_t)T * N * 4 + (size_t)T * DT * 4;
}
size_t bwd_smem(int T, int N, int esz) {
    const int DT = kRealDT, NT = real_threads(N);
    const int TB = T < kRealMaxTB ? T : kRealMaxTB;
    return (size_t)TB * DT * esz * 3 + (size_t)TB * N * 4 * 2 + (size_t)TB * DT * 4 +
           (size_t)(TB / kRealTS) * NT * 16 + (size_t)kRealTS * (NT / 32) * 2 * N * 4;
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename E, int N>
cudaError_t real_fwd_impl(const RealArgs& a, cudaStream_t st) {
    const dim3 block(real_threads(N));
    const size_t esz = sizeof(E);
    cudaError_t e;
    if (a.nseg > 1) {
        const size_t sm = fwd_smem(a.T, N, (int)esz);
        if ((e = set_smem(real_fwd_kernel<E, N, true>, sm)) != cudaSuccess) return e;
        real_fwd_kernel<E, N, true><<<dim3(a.ndt, a.B, a.nseg - 1), block, sm, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.D * N;
        real_carry_fwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.B, a.nseg, a.D * N,
                                                                            a.sumP, a.sumS, a.hin);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t sm = fwd_smem(a.T, N, (int)esz);
    if ((e = set_smem(real_fwd_kernel<E, N, false>, sm)) != cudaSuccess) return e;
    real_fwd_kernel<E, N, false><<<dim3(a.ndt, a.B, a.nseg), block, sm, st>>>(a);
    return cudaGetLastError();
}

template <typename E, int N>
cudaError_t real_bwd_impl(const RealArgs& a, cudaStream_t st) {
    const dim3 block(real_threads(N));
    const int esz = (int)sizeof(E);
    cudaError_t e;
    if (a.nseg > 1) {
        const size_t sm = bwd_summary_smem(a.T, N, esz);
        if ((e = set_smem(real_bwd_summary_kernel<E, N>, sm)) != cudaSuccess) return e;
        real_bwd_summary_kernel<E, N><<<dim3(a.ndt, a.B, a.nseg - 1), block, sm, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.D * N;
        real_carry_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.B, a.nseg, a.D * N,
                                                                            a.gsumP, a.gsumG, a.vin);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t sm = bwd_smem(a.T, N, esz);
    if ((e = set_smem(real_bwd_kernel<E, N>, sm)) != cudaSuccess) return e;
    real_bwd_kernel<E, N><<<dim3(a.ndt, a.B, a.nseg), block, sm, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t nbc = (int64_t)a.B * a.L * 2 * N;
    if (nbc > 0) {
        real_reduce_dbc_kernel<E, N><<<(unsigned)((nbc + 255) / 256), 256, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int64_t np = (int64_t)a.D * N;
    real_reduce_params_kernel<<<(unsigned)((np + 255) / 256), 256, 0, st>>>(a, N);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_real_fwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st) {
    if (io_bf16) {
        if (N == 4) return real_fwd_impl<__nv_bfloat16, 4>(a, st);
        if (N == 8) return real_fwd_impl<__nv_bfloat16, 8>(a, st);
        return real_fwd_impl<__nv_bfloat16, 16>(a, st);
    }
    if (N == 4) return real_fwd_impl<float, 4>(a, st);
    if (N == 8) return real_fwd_impl<float, 8>(a, st);
    return real_fwd_impl<float, 16>(a, st);
}

cudaError_t launch_real_bwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st) {
    if (io_bf16) {
        if (N == 4) return real_bwd_impl<__nv_bfloat16, 4>(a, st);
        if (N == 8) return real_bwd_impl<__nv_bfloat16, 8>(a, st);
        return real_bwd_impl<__nv_bfloat16, 16>(a, st);
    }
    if (N == 4) return real_bwd_impl<float, 4>(a, st);
    if (N == 8) return real_bwd_impl<float, 8>(a, st);
    return real_bwd_impl<float, 16>(a, st);
}

}  // namespace ssm
