// Complex-mode scan with shared retention / phase control ("SPARC: Shared Phase and Retention
// Control for Efficient Adaptive Spectral Recurrence", abstract):
//   s_t = softplus(r_t),  a_{t,k} = exp(-lambda_k s_t + i omega_k phi_t),  h_t = a_t h_{t-1} + u_t.
// The whole trajectory h is this mode's output, so the backward reads h_{t-1} from it rather than
// recomputing it, and sweeps the adjoint of Re sum conj(g) h backwards:
//   mu_t = g_t + w_{t+1},  w_t = conj(a_t) mu_t,  q_t = mu_t conj(a_t h_{t-1}) = w_t conj(h_{t-1}),
//   du = mu,  dlambda = -sum s Re q,  dr = sigmoid(r) (-sum_k lambda Re q),
//   domega = sum phi Im q,  dphi = sum_k omega Im q.
// Thread = one mode of one batch row; CTA = kCplxKT modes x one time segment.  Segments other than
// the first (forward) / last (backward) take their entering carry from a summary + carry pass,
// as in the real mode.
#include "ssm_device.cuh"
#include "ssm_internal.h"

namespace ssm {
namespace {

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// conj(a) * b
__device__ __forceinline__ float2 cmul_ca(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.x, b.y, -a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmul_cb(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}

// exp(-lam s + i om ph).  The phase product is split into its rounded value and exact residual
// (one fma), and the residual is applied to the sine/cosine to first order, so the phase carries
// no fp32 rounding of om*ph.
__device__ __forceinline__ float2 transition(float lam, float om, float s, float ph) {
    const float rho = expf(-lam * s);
    const float th = om * ph;
    const float tl = fmaf(om, ph, -th);
    float sn, cs;
    sincosf(th, &sn, &cs);
    const float c2 = fmaf(-tl, sn, cs);
    const float s2 = fmaf(tl, cs, sn);
    return make_float2(rho * c2, rho * s2);
}

template <bool SUMMARY>
__global__ void __launch_bounds__(kCplxKT) cplx_fwd_kernel(CplxArgs p) {
    constexpr int KT = kCplxKT, TT = kCplxTT;
    __shared__ __align__(16) float2 su[TT * KT];
    __shared__ float ss[TT], sph[TT];
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT, k = k0 + tid;
    const bool kv = k < p.K;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);
    const int TTe = min(TT, p.T);
    const float lam = kv ? p.lam[k] : 0.0f, om = kv ? p.om[k] : 0.0f;
    float2 h = make_float2(0.0f, 0.0f), P = make_float2(1.0f, 0.0f);
    if (!SUMMARY && seg > 0 && kv)
        h = reinterpret_cast<const float2*>(p.hin)[((size_t)b * p.nseg + seg) * p.K + k];
    const size_t boff = (size_t)b * p.L;
    const float2* ub = reinterpret_cast<const float2*>(p.u) + boff * p.K;
    float2* hb = SUMMARY ? nullptr : reinterpret_cast<float2*>(p.h) + boff * p.K;
    const float* rb = p.r + boff;
    const float* pb = p.phi + boff;

    for (int c = c_begin; c < c_end; ++c) {
        for (int sub = 0; sub < p.T; sub += TTe) {
            const int t0 = c * p.T + sub;
            if (t0 >= p.L) break;
            const int rows = min(TTe, p.L - t0);
            __syncthreads();
            load_tile<float2, KT>(su, ub, t0, rows, p.L, k0, p.K, tid, KT);
            if (tid < rows) {
                ss[tid] = softplus_acc(rb[t0 + tid]);
                sph[tid] = pb[t0 + tid];
            }
            __syncthreads();
            for (int r = 0; r < rows; ++r) {
                const float2 a = transition(lam, om, ss[r], sph[r]);
                const float2 uu = su[r * KT + tid];
                const float2 ah = cmul(a, h);
                h = make_float2(ah.x + uu.x, ah.y + uu.y);
                if (SUMMARY)
                    P = cmul(a, P);
                else
                    su[r * KT + tid] = h;
            }
            if (!SUMMARY) {
                __syncthreads();
                store_tile<float2, KT>(hb, su, t0, rows, p.L, k0, p.K, tid, KT);
            }
        }
    }
    if (SUMMARY) {
        if (kv) {
            const size_t o = ((size_t)b * (p.nseg - 1) + seg) * p.K + k;
            reinterpret_cast<float2*>(p.sumP)[o] = P;
            reinterpret_cast<float2*>(p.sumS)[o] = h;
        }
    } else if (kv && !(isfinite(h.x) && isfinite(h.y))) {
        flag_status(p.status, kStatusNonFinite);
    }
}

__global__ void cplx_carry_fwd_kernel(int B, int nseg, int K, const float2* __restrict__ P,
                                      const float2* __restrict__ Sv, float2* __restrict__ hin) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * K) return;
    const int b = (int)(i / K), k = (int)(i % K);
    float2 h = make_float2(0.0f, 0.0f);
    for (int s = 0; s < nseg; ++s) {
        hin[((size_t)b * nseg + s) * K + k] = h;
        if (s < nseg - 1) {
            const size_t j = ((size_t)b * (nseg - 1) + s) * K + k;
            const float2 ph = cmul(P[j], h);
            h = make_float2(ph.x + Sv[j].x, ph.y + Sv[j].y);
        }
    }
}

// Backward summary for segments 1..nseg-1: local reverse sweep from zero, w <- conj(a)(g + w),
// and P = prod conj(a) over the segment.
__global__ void __launch_bounds__(kCplxKT) cplx_bwd_summary_kernel(CplxArgs p) {
    constexpr int KT = kCplxKT, TT = kCplxTT;
    __shared__ __align__(16) float2 sg[TT * KT];
    __shared__ float ss[TT], sph[TT];
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT, k = k0 + tid;
    const bool kv = k < p.K;
    const int b = blockIdx.y, seg = blockIdx.z + 1;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);
    const int TTe = min(TT, p.T);
    const float lam = kv ? p.lam[k] : 0.0f, om = kv ? p.om[k] : 0.0f;
    float2 w = make_float2(0.0f, 0.0f), P = make_float2(1.0f, 0.0f);
    const size_t boff = (size_t)b * p.L;
    const float2* gb = reinterpret_cast<const float2*>(p.g) + boff * p.K;
    const float* rb = p.r + boff;
    const float* pb = p.phi + boff;
    for (int c = c_end - 1; c >= c_begin; --c) {
        for (int sub = ((p.T - 1) / TTe) * TTe; sub >= 0; sub -= TTe) {
            const int t0 = c * p.T + sub;
            if (t0 >= p.L) continue;
            const int rows = min(TTe, p.L - t0);
            __syncthreads();
            load_tile<float2, KT>(sg, gb, t0, rows, p.L, k0, p.K, tid, KT);
            if (tid < rows) {
                ss[tid] = softplus_acc(rb[t0 + tid]);
                sph[tid] = pb[t0 + tid];
            }
            __syncthreads();
            for (int r = rows - 1; r >= 0; --r) {
                const float2 a = transition(lam, om, ss[r], sph[r]);
                const float2 gg = sg[r * KT + tid];
                w = cmul_ca(a, make_float2(gg.x + w.x, gg.y + w.y));
                P = cmul_ca(a, P);
            }
        }
    }
    if (kv) {
        const size_t o = ((size_t)b * (p.nseg - 1) + (seg - 1)) * p.K + k;
        reinterpret_cast<float2*>(p.gsumP)[o] = P;
        reinterpret_cast<float2*>(p.gsumG)[o] = w;
    }
}

__global__ void cplx_carry_bwd_kernel(int B, int nseg, int K, const float2* __restrict__ P,
                                      const float2* __restrict__ G, float2* __restrict__ win) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * K) return;
    const int b = (int)(i / K), k = (int)(i % K);
    float2 w = make_float2(0.0f, 0.0f);
    for (int s = nseg - 1; s >= 0; --s) {
        win[((size_t)b * nseg + s) * K + k] = w;
        if (s > 0) {
            const size_t j = ((size_t)b * (nseg - 1) + (s - 1)) * K + k;
            const float2 pw = cmul(P[j], w);
            w = make_float2(pw.x + G[j].x, pw.y + G[j].y);
        }
    }
}

__global__ void __launch_bounds__(kCplxKT) cplx_bwd_kernel(CplxArgs p) {
    constexpr int KT = kCplxKT, TT = kCplxTT, NW = KT / 32;
    __shared__ __align__(16) float2 sg[TT * KT];   // g, then du in place
    __shared__ __align__(16) float2 shp[TT * KT];  // h_{t-1} for the tile's steps
    __shared__ float ss[TT], sph[TT];
    __shared__ float sred[TT * NW * 2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k0 = blockIdx.x * KT, k = k0 + tid;
    const bool kv = k < p.K;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);
    const int TTe = min(TT, p.T);
    const float lam = kv ? p.lam[k] : 0.0f, om = kv ? p.om[k] : 0.0f;
    float2 w = make_float2(0.0f, 0.0f);
    if (seg < p.nseg - 1 && kv)
        w = reinterpret_cast<const float2*>(p.win)[((size_t)b * p.nseg + seg) * p.K + k];
    float dlam = 0.0f, dom = 0.0f;
    const size_t boff = (size_t)b * p.L;
    const float2* gb = reinterpret_cast<const float2*>(p.g) + boff * p.K;
    const float2* hb = reinterpret_cast<const float2*>(p.h_in) + boff * p.K;
    float2* dub = reinterpret_cast<float2*>(p.du) + boff * p.K;
    const float* rb = p.r + boff;
    const float* pb = p.phi + boff;
    float* partb = p.rp_part + ((size_t)blockIdx.x * p.B + b) * (size_t)p.L * 2;

    for (int c = c_end - 1; c >= c_begin; --c) {
        for (int sub = ((p.T - 1) / TTe) * TTe; sub >= 0; sub -= TTe) {
            const int t0 = c * p.T + sub;
            if (t0 >= p.L) continue;
            const int rows = min(TTe, p.L - t0);
            __syncthreads();
            load_tile<float2, KT>(sg, gb, t0, rows, p.L, k0, p.K, tid, KT);
            if (t0 > 0) {
                load_tile<float2, KT>(shp, hb, t0 - 1, rows, p.L, k0, p.K, tid, KT);
            } else {
                shp[tid] = make_float2(0.0f, 0.0f);
                if (rows > 1) load_tile<float2, KT>(shp + KT, hb, 0, rows - 1, p.L, k0, p.K, tid, KT);
            }
            if (tid < rows) {
                ss[tid] = softplus_acc(rb[t0 + tid]);
                sph[tid] = pb[t0 + tid];
            }
            __syncthreads();
            for (int r = rows - 1; r >= 0; --r) {
                const float s = ss[r], ph = sph[r];
                const float2 a = transition(lam, om, s, ph);
                const float2 gg = sg[r * KT + tid];
                const float2 mu = make_float2(gg.x + w.x, gg.y + w.y);
                w = cmul_ca(a, mu);
                const float2 q = cmul_cb(w, shp[r * KT + tid]);
                sg[r * KT + tid] = mu;
                dlam = fmaf(-s, q.x, dlam);
                dom = fmaf(ph, q.y, dom);
                float rp = lam * q.x, pp = om * q.y;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    rp += __shfl_xor_sync(0xffffffffu, rp, o);
                    pp += __shfl_xor_sync(0xffffffffu, pp, o);
                }
                if (lane == 0) {
                    sred[(r * NW + warp) * 2 + 0] = rp;
                    sred[(r * NW + warp) * 2 + 1] = pp;
                }
            }
            __syncthreads();
            for (int i = tid; i < rows * 2; i += KT) {
                const int r = i >> 1, o = i & 1;
                float s = 0.0f;
#pragma unroll
                for (int ww = 0; ww < NW; ++ww) s += sred[(r * NW + ww) * 2 + o];
                partb[(size_t)(t0 + r) * 2 + o] = s;
            }
            store_tile<float2, KT>(dub, sg, t0, rows, p.L, k0, p.K, tid, KT);
        }
    }
    if (kv) {
        const size_t o = ((size_t)b * p.nseg + seg) * p.K + k;
        reinterpret_cast<float2*>(p.lo_part)[o] = make_float2(dlam, dom);
        if (!(isfinite(w.x) && isfinite(w.y))) flag_status(p.status, kStatusNonFinite);
    }
}

// dr = -sigmoid(r) * sum over mode tiles of sum_k lambda Re q;  dphi = sum of sum_k omega Im q.
__global__ void cplx_reduce_bl_kernel(CplxArgs p) {
    const int64_t n = (int64_t)p.B * p.L;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float sr = 0.0f, sp = 0.0f;
    for (int t = 0; t < p.nkt; ++t) {
        const float2 v = reinterpret_cast<const float2*>(p.rp_part)[(size_t)t * n + i];
        sr += v.x;
        sp += v.y;
    }
    p.dr[i] = -sigmoid_acc(p.r[i]) * sr;
    p.dphi[i] = sp;
}

__global__ void cplx_reduce_k_kernel(CplxArgs p) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= p.K) return;
    float sl = 0.0f, so = 0.0f;
    const int BS = p.B * p.nseg;
    for (int j = 0; j < BS; ++j) {
        const float2 v = reinterpret_cast<const float2*>(p.lo_part)[(size_t)j * p.K + k];
        sl += v.x;
        so += v.y;
    }
    p.dlam[k] = sl;
    p.dom[k] = so;
}

}  // namespace

cudaError_t launch_cplx_fwd(const CplxArgs& a, cudaStream_t st) {
    cudaError_t e;
    if (a.nseg > 1) {
        cplx_fwd_kernel<true><<<dim3(a.nkt, a.B, a.nseg - 1), kCplxKT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.K;
        cplx_carry_fwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            a.B, a.nseg, a.K, reinterpret_cast<const float2*>(a.sumP),
            reinterpret_cast<const float2*>(a.sumS), reinterpret_cast<float2*>(a.hin));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cplx_fwd_kernel<false><<<dim3(a.nkt, a.B, a.nseg), kCplxKT, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_cplx_bwd(const CplxArgs& a, cudaStream_t st) {
    cudaError_t e;
    if (a.nseg > 1) {
        cplx_bwd_summary_kernel<<<dim3(a.nkt, a.B, a.nseg - 1), kCplxKT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.K;
        cplx_carry_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            a.B, a.nseg, a.K, reinterpret_cast<const float2*>(a.gsumP),
            reinterpret_cast<const float2*>(a.gsumG), reinterpret_cast<float2*>(a.win));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cplx_bwd_kernel<<<dim3(a.nkt, a.B, a.nseg), kCplxKT, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t n = (int64_t)a.B * a.L;
    if (n > 0) {
        cplx_reduce_bl_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cplx_reduce_k_kernel<<<(a.K + 255) / 256, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ssm
