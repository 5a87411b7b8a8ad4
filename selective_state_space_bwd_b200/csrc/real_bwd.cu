// Real-mode exact backward: chunk recompute from checkpoints and reverse-time adjoint.
//
// Gradient of sum(dy * y) for the selective scan of real_fwd.cu ("Breaking the Memory Wall:
// Exact Analytical Differentiation via Tiled Operator-Space Evolution", abstract: exact analytical
// derivatives without materialising the graph; only chunk-end states are stored).  With
// g_t = dL/dh_t = C_t dy_t + a_{t+1} g_{t+1} and q_t = g_t a_t h_{t-1}:
//   dx = D dy + delta sum_n g B,  ddelta = sum_n A q + x sum_n g B,  ddelta_raw = ddelta sigmoid,
//   dB = sum_d g delta x,  dC = sum_d dy h,  dA_log = A sum_{b,t} delta q,  dD = sum_{b,t} dy x.
// Thread = (channel, S consecutive states), state pairs in packed fp32x2 arithmetic; NG = N / S
// adjacent lanes per channel; 32 channels per CTA; a CTA walks its time segment's chunks in
// reverse.  Time segments other than the last take their entering adjoint from a reverse
// summary + carry pass (three-phase structure of "Flash PD-SSM", technical summary).
#include "real_common.cuh"

namespace ssm {
namespace real {
namespace {

// ------------------------------------------------------------------------------------------------
// Backward segment summary (segments 1..nseg-1): local reverse adjoint from zero over the
// segment, v <- a_t (C_t dy_t + v), and P = prod a over the segment.
template <typename E, int N, int S>
__global__ void __launch_bounds__(RealCfg<N, S>::NT) real_bwd_summary_kernel(RealArgs p) {
    using Cfg = RealCfg<N, S>;
    constexpr int P2 = Cfg::P2, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT, U = Cfg::U;
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

    float2 A2[P2], v[P2], P[P2];
#pragma unroll
    for (int i = 0; i < P2; ++i) {
        A2[i] = dv ? make_float2(-expf(p.A_log[d * N + n0 + 2 * i]) * kLog2e,
                                 -expf(p.A_log[d * N + n0 + 2 * i + 1]) * kLog2e)
                   : make_float2(0.0f, 0.0f);
        v[i] = make_float2(0.0f, 0.0f);
        P[i] = make_float2(1.0f, 1.0f);
    }
    const size_t boff = (size_t)b * p.L;
    const E* dyb = static_cast<const E*>(p.dy) + boff * p.D;
    const E* drb = static_cast<const E*>(p.draw) + boff * p.D;
    const E* Cb = static_cast<const E*>(p.Cm) + boff * N;

    for (int c = c_end - 1; c >= c_begin; --c) {
        const int t0 = c * T;
        const int rows = min(T, p.L - t0);
        const int rows4 = (rows + U - 1) / U * U;
        __syncthreads();
        load_tile<E, DT>(sdy, dyb, t0, rows4, p.L, d0, p.D, tid, NT);
        load_tile<E, DT>(sdr, drb, t0, rows4, p.L, d0, p.D, tid, NT);
        load_rows_f32<E, N>(sC, Cb, t0, rows4, p.L, tid, NT);
        __syncthreads();
        for (int i = tid; i < rows4 * DT; i += NT)
            sdel[i] = i < rows * DT ? softplus_fast(Elem<E>::to_f(sdr[i])) : 0.0f;
        __syncthreads();
        for (int r0 = rows4 - U; r0 >= 0; r0 -= U) {
#pragma unroll
            for (int u = U - 1; u >= 0; --u) {
                const int r = r0 + u;
                const float dlt = sdel[r * DT + dl];
                const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                float2 cq[P2];
                ld_pairs<S>(cq, sC + r * N + n0);
#pragma unroll
                for (int i = 0; i < P2; ++i) {
                    const float2 a = ex2_pair(__fmul2_rn(f2(dlt), A2[i]));
                    v[i] = __fmul2_rn(a, __ffma2_rn(cq[i], f2(dyv), v[i]));
                    P[i] = __fmul2_rn(P[i], a);
                }
            }
        }
    }
    if (dv) {
        const size_t o = (((size_t)b * (p.nseg - 1) + (seg - 1)) * p.D + d) * N + n0;
        st_pairs<S>(p.gsumP + o, P);
        st_pairs<S>(p.gsumG + o, v);
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

// ------------------------------------------------------------------------------------------------
// Backward main kernel.  For every stretch of TB <= 128 steps (a chunk, or half a 256-step
// chunk), in reverse order:
//   pass A: recompute h forward from the chunk checkpoint; the state at the start of every
//           TS-step window goes to an L2-resident scratch region owned by this CTA;
//   pass B: for each window in reverse, recompute (a_t, a_t h_{t-1}) into registers and sweep
//           the adjoint backwards in groups of 4 steps, emitting dx and ddelta_raw per channel,
//           the sums of dB and dC over the CTA's 32 channels, and per-thread sums for dA_log, dD.
// Shared memory: x, delta_raw, dy raw tiles [TB][DT] (x's and delta_raw's reused for dx and
// ddelta_raw); B, C float [TB][N]; delta [TB][DT]; dB/dC values of one 4-step group [4][DT][2N].
template <typename E, int N, int S>
__global__ void __launch_bounds__(RealCfg<N, S>::NT) real_bwd_kernel(RealArgs p) {
    using Cfg = RealCfg<N, S>;
    constexpr int P2 = Cfg::P2, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT, TS = Cfg::TS;
    constexpr int U = Cfg::U, Q = Cfg::Q, N2 = 2 * N;
    extern __shared__ __align__(16) unsigned char smem[];
    const int T = p.T;
    const int TB = min(T, kRealMaxTB);
    E* sx = reinterpret_cast<E*>(smem);
    E* sdr = sx + TB * DT;
    E* sdy = sdr + TB * DT;
    float* sB = reinterpret_cast<float*>(sdy + TB * DT);
    float* sC = sB + TB * N;
    float* sdel = sC + TB * N;
    float* sred = sdel + TB * DT;

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * S;
    const bool dv = d < p.D;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);
    // column-sum roles: `part` sums channels [part*DT/Q, ...) of output quad `quad`
    const int cs_part = (tid >> 3) % Q;
    const int cs_quad = (tid & 7) + 8 * (tid / (8 * Q));
    const int cs_u = cs_quad / (N2 / 4), cs_o = 4 * (cs_quad % (N2 / 4));

    float2 A[P2], A2[P2], v[P2], dA[P2];
#pragma unroll
    for (int i = 0; i < P2; ++i) {
        A[i] = dv ? make_float2(-expf(p.A_log[d * N + n0 + 2 * i]), -expf(p.A_log[d * N + n0 + 2 * i + 1]))
                  : make_float2(0.0f, 0.0f);
        A2[i] = __fmul2_rn(A[i], f2(kLog2e));
        v[i] = make_float2(0.0f, 0.0f);
        dA[i] = make_float2(0.0f, 0.0f);
    }
    if (seg < p.nseg - 1 && dv) ld_pairs<S>(v, p.vin + (((size_t)b * p.nseg + seg) * p.D + d) * N + n0);
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
    const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    float* bnd = p.bnd_scratch + cta * (size_t)(kRealMaxTB / TS) * NT * S + (size_t)tid * S;

    const int per_chunk = T / TB;  // 1, or 2 for 256-step chunks
    for (int c = c_end - 1; c >= c_begin; --c) {
        for (int part = per_chunk - 1; part >= 0; --part) {
            const int t0 = c * T + part * TB;
            if (t0 >= p.L) continue;
            const int rows = min(TB, p.L - t0);
            const int rows4 = (rows + U - 1) / U * U;
            // state entering this stretch
            float2 h[P2];
            if (c > 0 && dv) {
                ld_pairs<S>(h, p.ckpt_in + (((size_t)b * p.nC + (c - 1)) * p.D + d) * N + n0);
            } else {
#pragma unroll
                for (int i = 0; i < P2; ++i) h[i] = make_float2(0.0f, 0.0f);
            }
            for (int pre = 0; pre < part; ++pre) {  // advance through the chunk's earlier stretch
                const int tp = c * T + pre * TB;
                __syncthreads();
                load_tile<E, DT>(sx, xb, tp, TB, p.L, d0, p.D, tid, NT);
                load_tile<E, DT>(sdr, drb, tp, TB, p.L, d0, p.D, tid, NT);
                load_rows_f32<E, N>(sB, Bb, tp, TB, p.L, tid, NT);
                __syncthreads();
                for (int r = 0; r < TB; ++r) {
                    const float dlt = softplus_fast(Elem<E>::to_f(sdr[r * DT + dl]));
                    const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                    float2 bq[P2];
                    ld_pairs<S>(bq, sB + r * N + n0);
#pragma unroll
                    for (int i = 0; i < P2; ++i)
                        h[i] = __ffma2_rn(ex2_pair(__fmul2_rn(f2(dlt), A2[i])), h[i], __fmul2_rn(f2(dxv), bq[i]));
                }
            }
            __syncthreads();
            load_tile<E, DT>(sx, xb, t0, rows4, p.L, d0, p.D, tid, NT);
            load_tile<E, DT>(sdr, drb, t0, rows4, p.L, d0, p.D, tid, NT);
            load_tile<E, DT>(sdy, dyb, t0, rows4, p.L, d0, p.D, tid, NT);
            load_rows_f32<E, N>(sB, Bb, t0, rows4, p.L, tid, NT);
            load_rows_f32<E, N>(sC, Cb, t0, rows4, p.L, tid, NT);
            __syncthreads();
            // steps past the sequence end get delta = 0 (a = 1, no input): they pass state and
            // adjoint through unchanged
            for (int i = tid; i < rows4 * DT; i += NT)
                sdel[i] = i < rows * DT ? softplus_fast(Elem<E>::to_f(sdr[i])) : 0.0f;
            __syncthreads();

            // pass A
            const int nwin = (rows4 + TS - 1) / TS;
            for (int k = 0; k < nwin; ++k) {
                st_pairs_cg<S>(bnd + (size_t)k * NT * S, h);
#pragma unroll
                for (int ts = 0; ts < TS; ++ts) {
                    const int r = k * TS + ts;
                    if (TS > U && r >= rows4) break;
                    const float dlt = sdel[r * DT + dl];
                    const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                    float2 bq[P2];
                    ld_pairs<S>(bq, sB + r * N + n0);
#pragma unroll
                    for (int i = 0; i < P2; ++i)
                        h[i] = __ffma2_rn(ex2_pair(__fmul2_rn(f2(dlt), A2[i])), h[i], __fmul2_rn(f2(dxv), bq[i]));
                }
            }

            // pass B
            float2 hw[P2];
            ld_pairs_cg<S>(hw, bnd + (size_t)(nwin - 1) * NT * S);
            for (int k = nwin - 1; k >= 0; --k) {
                float2 aa[TS][P2], pp[TS][P2];
                {
                    float2 hc[P2];
#pragma unroll
                    for (int i = 0; i < P2; ++i) hc[i] = hw[i];
                    if (k > 0) ld_pairs_cg<S>(hw, bnd + (size_t)(k - 1) * NT * S);  // prefetch
#pragma unroll
                    for (int ts = 0; ts < TS; ++ts) {
                        const int r = k * TS + ts;
                        const float dlt = (TS > U && r >= rows4) ? 0.0f : sdel[r * DT + dl];
                        const float dxv = (TS > U && r >= rows4) ? 0.0f : dlt * Elem<E>::to_f(sx[r * DT + dl]);
                        float2 bq[P2];
                        if (TS > U && r >= rows4) {
#pragma unroll
                            for (int i = 0; i < P2; ++i) bq[i] = make_float2(0.0f, 0.0f);
                        } else {
                            ld_pairs<S>(bq, sB + r * N + n0);
                        }
#pragma unroll
                        for (int i = 0; i < P2; ++i) {
                            const float2 a = ex2_pair(__fmul2_rn(f2(dlt), A2[i]));
                            const float2 pr = __fmul2_rn(a, hc[i]);
                            aa[ts][i] = a;
                            pp[ts][i] = pr;
                            hc[i] = __ffma2_rn(f2(dxv), bq[i], pr);
                        }
                    }
                }
#pragma unroll
                for (int g4 = TS / U - 1; g4 >= 0; --g4) {
                    const int rg = k * TS + g4 * U;
                    if (TS > U && rg >= rows4) continue;
                    float sv[2 * U];
#pragma unroll
                    for (int u = U - 1; u >= 0; --u) {
                        const int ts = g4 * U + u;
                        const int r = rg + u;
                        const float dlt = sdel[r * DT + dl];
                        const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                        const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                        float2 bq[P2], cq[P2];
                        ld_pairs<S>(bq, sB + r * N + n0);
                        ld_pairs<S>(cq, sC + r * N + n0);
                        float2 sg = make_float2(0.0f, 0.0f), sa = make_float2(0.0f, 0.0f);
                        float2 rB[P2], rC[P2];
#pragma unroll
                        for (int i = 0; i < P2; ++i) {
                            const float2 g = __ffma2_rn(cq[i], f2(dyv), v[i]);
                            const float2 hj = __ffma2_rn(f2(dxv), bq[i], pp[ts][i]);
                            const float2 q = __fmul2_rn(g, pp[ts][i]);
                            dA[i] = __ffma2_rn(f2(dlt), q, dA[i]);
                            sa = __ffma2_rn(A[i], q, sa);
                            sg = __ffma2_rn(g, bq[i], sg);
                            rB[i] = __fmul2_rn(g, f2(dxv));
                            rC[i] = __fmul2_rn(f2(dyv), hj);
                            v[i] = __fmul2_rn(aa[ts][i], g);
                        }
                        sv[2 * u] = sg.x + sg.y;
                        sv[2 * u + 1] = sa.x + sa.y;
                        float* sr = sred + (u * DT + dl) * N2 + n0;
                        st_pairs<S>(sr, rB);
                        st_pairs<S>(sr + N, rC);
                    }
                    // per-channel sums over the NG lanes: lane ng gets steps [ng*U/NG, ...)
                    reduce_scatter<2 * U, NG>(sv, ng);
#pragma unroll
                    for (int j = 0; j < U / NG; ++j) {
                        const int r = rg + ng * (U / NG) + j;
                        if (r < rows) {
                            const float dlt = sdel[r * DT + dl];
                            const float xv = Elem<E>::to_f(sx[r * DT + dl]);
                            const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                            const float sgB = sv[2 * j], sAq = sv[2 * j + 1];
                            const float sig = sigmoid_fast(Elem<E>::to_f(sdr[r * DT + dl]));
                            sx[r * DT + dl] = Elem<E>::from_f(fmaf(dsk, dyv, dlt * sgB));
                            sdr[r * DT + dl] = Elem<E>::from_f(fmaf(xv, sgB, sAq) * sig);
                            dDacc = fmaf(dyv, xv, dDacc);
                        }
                    }
                    __syncthreads();
                    {   // dB, dC: sum the group's values over the CTA's channels
                        const float* src = sred + (cs_u * DT + cs_part * (DT / Q)) * N2 + cs_o;
                        float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0, s3 = s0;
#pragma unroll
                        for (int ch = 0; ch < DT / Q; ch += 2) {
                            const float4 a0 = *reinterpret_cast<const float4*>(src + ch * N2);
                            const float4 a1 = *reinterpret_cast<const float4*>(src + (ch + 1) * N2);
                            s0 = __fadd2_rn(s0, make_float2(a0.x, a0.y));
                            s1 = __fadd2_rn(s1, make_float2(a0.z, a0.w));
                            s2 = __fadd2_rn(s2, make_float2(a1.x, a1.y));
                            s3 = __fadd2_rn(s3, make_float2(a1.z, a1.w));
                        }
                        s0 = __fadd2_rn(s0, s2);
                        s1 = __fadd2_rn(s1, s3);
#pragma unroll
                        for (int m = 8; m < 8 * Q; m <<= 1) {
                            s0.x += __shfl_xor_sync(kFull, s0.x, m);
                            s0.y += __shfl_xor_sync(kFull, s0.y, m);
                            s1.x += __shfl_xor_sync(kFull, s1.x, m);
                            s1.y += __shfl_xor_sync(kFull, s1.y, m);
                        }
                        const int r = rg + cs_u;
                        if (cs_part == 0 && r < rows)
                            *reinterpret_cast<float4*>(partb + (size_t)(t0 + r) * N2 + cs_o) =
                                make_float4(s0.x, s0.y, s1.x, s1.y);
                    }
                    __syncthreads();
                }
            }
            store_tile<E, DT>(dxb, sx, t0, rows, p.L, d0, p.D, tid, NT);
            store_tile<E, DT>(ddrb, sdr, t0, rows, p.L, d0, p.D, tid, NT);
        }
    }
    // each lane of a channel accumulated dD over its own subset of steps
#pragma unroll
    for (int m = 1; m < NG; m <<= 1) dDacc += __shfl_xor_sync(kFull, dDacc, m);
    if (dv) {
        const size_t o = (((size_t)b * p.nseg + seg) * p.D + d) * N + n0;
        st_pairs<S>(p.dA_part + o, dA);
        if (ng == 0) p.dD_part[((size_t)b * p.nseg + seg) * p.D + d] = dDacc;
        if (!all_finite<S>(v)) flag_status(p.status, kStatusNonFinite);
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

template <int N, int S>
size_t bwd_summary_smem(int T, int esz) {
    return (size_t)T * kRealDT * esz * 2 + (size_t)T * N * 4 + (size_t)T * kRealDT * 4;
}
template <int N, int S>
size_t bwd_smem(int T, int esz) {
    const int TB = T < kRealMaxTB ? T : kRealMaxTB;
    return (size_t)TB * kRealDT * esz * 3 + (size_t)TB * N * 4 * 2 + (size_t)TB * kRealDT * 4 +
           (size_t)RealCfg<N, S>::U * kRealDT * 2 * N * 4;
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename E, int N, int S>
cudaError_t real_bwd_impl(const RealArgs& a, cudaStream_t st) {
    const dim3 block(RealCfg<N, S>::NT);
    const int esz = (int)sizeof(E);
    cudaError_t e;
    if (a.nseg > 1) {
        const size_t sm = bwd_summary_smem<N, S>(a.T, esz);
        if ((e = set_smem(real_bwd_summary_kernel<E, N, S>, sm)) != cudaSuccess) return e;
        real_bwd_summary_kernel<E, N, S><<<dim3(a.ndt, a.B, a.nseg - 1), block, sm, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.D * N;
        real_carry_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.B, a.nseg, a.D * N,
                                                                            a.gsumP, a.gsumG, a.vin);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t sm = bwd_smem<N, S>(a.T, esz);
    if ((e = set_smem(real_bwd_kernel<E, N, S>, sm)) != cudaSuccess) return e;
    real_bwd_kernel<E, N, S><<<dim3(a.ndt, a.B, a.nseg), block, sm, st>>>(a);
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

template <typename E>
cudaError_t bwd_dispatch(const RealArgs& a, int N, cudaStream_t st) {
    if (N == 4) return real_bwd_impl<E, 4, 4>(a, st);
    if (N == 8) return real_bwd_impl<E, 8, kRealStates8>(a, st);
    return real_bwd_impl<E, 16, kRealStates16>(a, st);
}

}  // namespace
}  // namespace real

cudaError_t launch_real_bwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st) {
    return io_bf16 ? real::bwd_dispatch<__nv_bfloat16>(a, N, st) : real::bwd_dispatch<float>(a, N, st);
}

}  // namespace ssm
