// Complex-mode scan with shared retention / phase control ("SPARC: Shared Phase and Retention
// Control for Efficient Adaptive Spectral Recurrence", abstract):
//   s_t = softplus(r_t),  a_{t,k} = exp(-lambda_k s_t + i omega_k phi_t),  h_t = a_t h_{t-1} + u_t.
// The whole trajectory h is this mode's output, so the backward reads h_{t-1} from it rather than
// recomputing it, and sweeps the adjoint of Re sum conj(g) h backwards:
//   mu_t = g_t + w_{t+1},  w_t = conj(a_t) mu_t,  q_t = mu_t conj(a_t h_{t-1}) = w_t conj(h_{t-1}),
//   du = mu,  dlambda = -sum s Re q,  dr = sigmoid(r) (-sum_k lambda Re q),
//   domega = sum phi Im q,  dphi = sum_k omega Im q.
// A CTA takes kCplxKT modes of one batch row over one time segment and is warp-specialised: one
// consumer thread per mode runs the recurrence (or the adjoint sweep) over 16-step tiles streamed
// through its own cp.async ring, while two producer threads per mode compute the next tile's
// transitions a = exp(-lambda s + i omega phi) (an exp2 and a sine/cosine per update, most of
// the arithmetic, independent of the state) into one of two shared buffers, handed over with
// named barriers (the barrier sequences of both roles are model-checked on the host by
// tests/test_barrier_protocol.py).  The per-step sums over the modes (dr, dphi) go through
// shared memory, one column per step.  Segments other than the first (forward) / last
// (backward) take their entering carry from a summary + carry pass, as in the real mode.
#include "real_common.cuh"

namespace ssm {
namespace {

using real::cp_async_commit;
using real::cp_async_flat;
using real::cp_async_tile;
using real::cp_async_wait;

constexpr int KT = kCplxKT;
constexpr int TTF = kCplxTT;   // forward tile: steps per stage
constexpr int CB = 8;          // transitions computed together (independent of the state)

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

// sin and cos of a phase th.  Reduction by pi/2 with pi/2 split into three floats (the first two
// carry 12 significant bits, so kq times either is exact while |kq| < 4096), then the Taylor
// series of sin (to x^9) and cos (to x^10) on [-pi/4, pi/4], whose remainders are below 2e-9 and
// 1.1e-10 there.  Branch-free; `far` reports |th| beyond the reduction's range (|th| > ~6400),
// where the result is not used (see transitions()).
__device__ __forceinline__ void sincos_phase(float th, float& sn, float& cs, bool& far) {
    const float kq = rintf(th * 0x1.45f306p-1f);  // th * 2/pi
    far = fabsf(kq) >= 4096.0f;
    float x = fmaf(-kq, 0x1.92p+0f, th);
    x = fmaf(-kq, 0x1.fb4p-12f, x);
    x = fmaf(-kq, 0x1.4442d2p-24f, x);
    const float x2 = x * x;
    float ps = fmaf(x2, 1.0f / 362880.0f, -1.0f / 5040.0f);
    ps = fmaf(x2, ps, 1.0f / 120.0f);
    ps = fmaf(x2, ps, -1.0f / 6.0f);
    const float s = fmaf(x * x2, ps, x);
    float pc = fmaf(x2, -1.0f / 3628800.0f, 1.0f / 40320.0f);
    pc = fmaf(x2, pc, -1.0f / 720.0f);
    pc = fmaf(x2, pc, 1.0f / 24.0f);
    pc = fmaf(x2, pc, -0.5f);
    const float c = fmaf(x2, pc, 1.0f);
    const int q = static_cast<int>(kq) & 3;
    sn = q == 0 ? s : (q == 1 ? c : (q == 2 ? -s : -c));
    cs = q == 0 ? c : (q == 1 ? -s : (q == 2 ? -c : s));
}

// exp(-lam s + i om ph) from given sin/cos of the rounded phase th = om*ph; lam2 = lam log2(e).  The exact residual
// of the phase product (one fma) is applied to the sine/cosine to first order, so the phase
// carries no fp32 rounding of om*ph.
__device__ __forceinline__ float2 transition_from(float lam2, float om, float s, float ph, float th,
                                                  float sn, float cs) {
    const float rho = ex2_mufu(-lam2 * s);
    const float tl = fmaf(om, ph, -th);
    const float c2 = fmaf(-tl, sn, cs);
    const float s2 = fmaf(tl, cs, sn);
    return make_float2(rho * c2, rho * s2);
}

// The transitions a_{t,k} of CB consecutive steps (ss/sph at r0..r0+CB-1), computed together:
// they do not depend on the state, so their arithmetic overlaps.  Phases out of the reduction's
// range (never for |omega phi| < 6400) are redone with the library sincosf, warp-uniformly.
template <int CB, int STRIDE = 1>
__device__ __forceinline__ void transitions(float2 (&a)[CB], float lam2, float om,
                                            const float2* ssp, int r0) {
    bool any_far = false;
#pragma unroll
    for (int u = 0; u < CB; ++u) {
        const float2 sp = ssp[r0 + STRIDE * u];  // (s, phi)
        const float th = om * sp.y;
        float sn, cs;
        bool far;
        sincos_phase(th, sn, cs, far);
        any_far |= far;
        a[u] = transition_from(lam2, om, sp.x, sp.y, th, sn, cs);
    }
    if (__any_sync(0xffffffffu, any_far)) {
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const float2 sp = ssp[r0 + STRIDE * u];
            const float th = om * sp.y;
            if (fabsf(rintf(th * 0x1.45f306p-1f)) >= 4096.0f) {
                float sn, cs;
                sincosf(th, &sn, &cs);
                a[u] = transition_from(lam2, om, sp.x, sp.y, th, sn, cs);
            }
        }
    }
}

// The same transitions, two steps per packed fp32x2 operation (the producers' path): the
// reduction, both polynomials, the residual rotation and the decay exponent run as FFMA2 / FMUL2
// on (step u, step u+1), component by component the same roundings as transitions(), so the
// results are identical; the quadrant selection stays scalar.
template <int CB, int STRIDE>
__device__ __forceinline__ void transitions_pk(float2 (&a)[CB], float lam2, float om,
                                               const float2* ssp, int r0) {
    static_assert(CB % 2 == 0, "steps in pairs");
    using real::f2;
    bool any_far = false;
#pragma unroll
    for (int u = 0; u < CB; u += 2) {
        const float2 sp0 = ssp[r0 + STRIDE * u], sp1 = ssp[r0 + STRIDE * (u + 1)];  // (s, phi)
        const float2 ph = make_float2(sp0.y, sp1.y);
        const float2 th = __fmul2_rn(f2(om), ph);
        const float2 tq = __fmul2_rn(th, f2(0x1.45f306p-1f));  // th * 2/pi
        const float2 kq = make_float2(rintf(tq.x), rintf(tq.y));
        any_far |= fabsf(kq.x) >= 4096.0f || fabsf(kq.y) >= 4096.0f;
        const float2 nk = make_float2(-kq.x, -kq.y);
        float2 x = __ffma2_rn(nk, f2(0x1.92p+0f), th);
        x = __ffma2_rn(nk, f2(0x1.fb4p-12f), x);
        x = __ffma2_rn(nk, f2(0x1.4442d2p-24f), x);
        const float2 x2 = __fmul2_rn(x, x);
        float2 ps = __ffma2_rn(x2, f2(1.0f / 362880.0f), f2(-1.0f / 5040.0f));
        ps = __ffma2_rn(x2, ps, f2(1.0f / 120.0f));
        ps = __ffma2_rn(x2, ps, f2(-1.0f / 6.0f));
        const float2 sv = __ffma2_rn(__fmul2_rn(x, x2), ps, x);
        float2 pc = __ffma2_rn(x2, f2(-1.0f / 3628800.0f), f2(1.0f / 40320.0f));
        pc = __ffma2_rn(x2, pc, f2(-1.0f / 720.0f));
        pc = __ffma2_rn(x2, pc, f2(1.0f / 24.0f));
        pc = __ffma2_rn(x2, pc, f2(-0.5f));
        const float2 cv = __ffma2_rn(x2, pc, f2(1.0f));
        float2 sn, cs;
        {
            const int q = static_cast<int>(kq.x) & 3;
            sn.x = q == 0 ? sv.x : (q == 1 ? cv.x : (q == 2 ? -sv.x : -cv.x));
            cs.x = q == 0 ? cv.x : (q == 1 ? -sv.x : (q == 2 ? -cv.x : sv.x));
        }
        {
            const int q = static_cast<int>(kq.y) & 3;
            sn.y = q == 0 ? sv.y : (q == 1 ? cv.y : (q == 2 ? -sv.y : -cv.y));
            cs.y = q == 0 ? cv.y : (q == 1 ? -sv.y : (q == 2 ? -cv.y : sv.y));
        }
        const float2 ls = __fmul2_rn(f2(-lam2), make_float2(sp0.x, sp1.x));
        const float2 rho = make_float2(ex2_mufu(ls.x), ex2_mufu(ls.y));
        const float2 tl = __ffma2_rn(f2(om), ph, make_float2(-th.x, -th.y));
        const float2 c2 = __ffma2_rn(make_float2(-tl.x, -tl.y), sn, cs);
        const float2 s2 = __ffma2_rn(tl, cs, sn);
        a[u] = make_float2(rho.x * c2.x, rho.x * s2.x);
        a[u + 1] = make_float2(rho.y * c2.y, rho.y * s2.y);
    }
    if (__any_sync(0xffffffffu, any_far)) {
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const float2 sp = ssp[r0 + STRIDE * u];
            const float th = om * sp.y;
            if (fabsf(rintf(th * 0x1.45f306p-1f)) >= 4096.0f) {
                float sn, cs;
                sincosf(th, &sn, &cs);
                a[u] = transition_from(lam2, om, sp.x, sp.y, th, sn, cs);
            }
        }
    }
}

// Per-step scalars of a staged tile: s = softplus(r) and phi, for `rows` steps.
__device__ __forceinline__ void step_scalars(const float* sr, const float* sp, float2* ssp,
                                             int rows, int tid) {
    if (tid < rows) ssp[tid] = make_float2(softplus_acc(sr[tid]), sp[tid]);
}

// Forward, warp-specialised.  A CTA takes KT modes of one batch row over one time segment:
// KT consumer threads (one per mode) run the recurrence h = a h + u, and 2 KT producer threads
// (two per mode, alternate steps) compute the transitions a of the next 16-step tile into one of
// two shared buffers.  The transitions (an exp2 and a sine/cosine per update, most of the
// arithmetic) do not depend on the state, so the producers run ahead while the consumers' short
// dependent chain and HBM stream proceed; FULL / EMPTY named barriers hand the buffers over.
// SUMMARY = true: local scan from zero over segments 0..nseg-2, emitting (prod a, end state).
// SUMMARY = false: the scan from the segment's entering state, writing h.
constexpr int FT = 16;                 // steps per tile (divides every chunk length)
constexpr int F_CONS = KT;             // consumer threads
constexpr int F_PROD = 2 * KT;         // producer threads
constexpr int F_NT = F_CONS + F_PROD;
constexpr int F_USTAGES = 3;           // u ring of the consumers
constexpr int F_BAR_FULL = 1, F_BAR_EMPTY = 3, F_BAR_PROD = 5, F_BAR_CONS = 6;

__device__ __forceinline__ void bar_sync_n(int id, int n) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_arrive_n(int id, int n) {
    asm volatile("bar.arrive %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

template <bool SUMMARY>
__global__ void __launch_bounds__(F_NT) cplx_fwd_kernel(CplxArgs p) {
    __shared__ __align__(16) float2 sa[2][FT * KT];           // transitions of a tile
    __shared__ __align__(16) float2 su[F_USTAGES][FT * KT];   // u of a tile
    __shared__ float2 ssp[2][FT];                             // (softplus(r), phi) per step
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int t_begin = seg * p.seg_chunks * p.T;
    const int t_end = min(p.L, min(p.nC, (seg + 1) * p.seg_chunks) * p.T);
    const int ntiles = (t_end - t_begin + FT - 1) / FT;
    const size_t boff = (size_t)b * p.L;

    if (tid >= F_CONS) {
        // ---------------------------------------------------------------- producers
        const int pt = tid - F_CONS, kk = pt % KT, rp = pt / KT;  // mode, row parity
        const int k = k0 + kk;
        const bool kv = k < p.K;
        const float lam2 = kv ? p.lam[k] * kLog2e : 0.0f, om = kv ? p.om[k] : 0.0f;
        const float* rb = p.r + boff;
        const float* pb = p.phi + boff;
        // the step scalars of tile i + 1 are fetched while tile i is computed
        float rn = 0.0f, pn = 0.0f;
        if (pt < FT && t_begin + pt < t_end) {
            rn = rb[t_begin + pt];
            pn = pb[t_begin + pt];
        }
        for (int i = 0; i < ntiles; ++i) {
            const int buf = i & 1;
            const int t0 = t_begin + i * FT, rows = min(FT, t_end - t0);
            if (pt < FT) {
                ssp[buf][pt] = pt < rows ? make_float2(softplus_acc(rn), pn) : make_float2(0.0f, 0.0f);
                const int tn = t0 + FT + pt;
                if (i + 1 < ntiles && tn < t_end) {
                    rn = rb[tn];
                    pn = pb[tn];
                }
            }
            bar_sync_n(F_BAR_PROD, F_PROD);               // the step scalars are in
            bar_sync_n(F_BAR_EMPTY + buf, F_NT);          // the consumers are done with buffer buf
            float2 a[FT / 2];
            transitions_pk<FT / 2, 2>(a, lam2, om, ssp[buf], rp);
#pragma unroll
            for (int u = 0; u < FT / 2; ++u) sa[buf][(rp + 2 * u) * KT + kk] = a[u];
            bar_arrive_n(F_BAR_FULL + buf, F_NT);         // buffer buf holds the tile's transitions
        }
        bar_sync_n(F_BAR_EMPTY + 0, F_NT);  // balance the consumers' last two releases
        bar_sync_n(F_BAR_EMPTY + 1, F_NT);
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int k = k0 + tid;
    const bool kv = k < p.K;
    float2 h = make_float2(0.0f, 0.0f), P = make_float2(1.0f, 0.0f);
    if (!SUMMARY && seg > 0 && kv)
        h = reinterpret_cast<const float2*>(p.hin)[((size_t)b * p.nseg + seg) * p.K + k];
    const float2* ub = reinterpret_cast<const float2*>(p.u) + boff * p.K;
    float2* hb = SUMMARY || !p.h ? nullptr : reinterpret_cast<float2*>(p.h) + boff * p.K;
    auto issue = [&](int i) {
        if (i < ntiles)
            cp_async_tile<float2, KT>(su[i % F_USTAGES], ub, t_begin + i * FT, FT, p.L, k0, p.K, tid,
                                      F_CONS);
        cp_async_commit();
    };
    issue(0);
    issue(1);
    bar_arrive_n(F_BAR_EMPTY + 0, F_NT);  // both transition buffers start empty
    bar_arrive_n(F_BAR_EMPTY + 1, F_NT);
    for (int i = 0; i < ntiles; ++i) {
        const int buf = i & 1;
        const int t0 = t_begin + i * FT, rows = min(FT, t_end - t0);
        cp_async_wait<F_USTAGES - 2>();
        bar_sync_n(F_BAR_CONS, F_CONS);  // u of tile i is in; both consumer warps are past tile i-1
        issue(i + 2);
        const float2* sut = su[i % F_USTAGES];
        const float2* sat = sa[buf];
        bar_sync_n(F_BAR_FULL + buf, F_NT);  // the producers have written the tile's transitions
#pragma unroll 4
        for (int r = 0; r < rows; ++r) {
            const float2 av = sat[r * KT + tid];
            const float2 uu = sut[r * KT + tid];
            const float2 ah = cmul(av, h);
            h = make_float2(ah.x + uu.x, ah.y + uu.y);
            if (SUMMARY)
                P = cmul(av, P);
            else if (kv && hb)
                hb[(size_t)(t0 + r) * p.K + k] = h;
        }
        bar_arrive_n(F_BAR_EMPTY + buf, F_NT);  // buffer buf is consumed
        // tiles never cross a chunk end (FT divides T): the state after the tile's last step is
        // the chunk's checkpoint when the tile ends the chunk
        const int te = t0 + rows;
        if (!SUMMARY && p.ckpt && kv && (te % p.T == 0 || te == p.L))
            reinterpret_cast<float2*>(p.ckpt)[((size_t)b * p.nC + (te - 1) / p.T) * p.K + k] = h;
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
__global__ void __launch_bounds__(KT) cplx_bwd_summary_kernel(CplxArgs p) {
    __shared__ __align__(16) float2 sg[2][TTF * KT];
    __shared__ __align__(16) float sr[2][TTF], sp[2][TTF];
    __shared__ float2 ssp[TTF];  // (softplus(r), phi) per step
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT, k = k0 + tid;
    const bool kv = k < p.K;
    const int b = blockIdx.y, seg = blockIdx.z + 1;
    const int TT = min(TTF, p.T);
    const int t_begin = seg * p.seg_chunks * p.T;
    const int t_end = min(p.L, min(p.nC, (seg + 1) * p.seg_chunks) * p.T);
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    const float lam = kv ? p.lam[k] : 0.0f, om = kv ? p.om[k] : 0.0f;
    float2 w = make_float2(0.0f, 0.0f), P = make_float2(1.0f, 0.0f);
    const size_t boff = (size_t)b * p.L;
    const float2* gb = reinterpret_cast<const float2*>(p.g) + boff * p.K;
    const float* rb = p.r + boff;
    const float* pb = p.phi + boff;
    auto issue = [&](int j, int st) {
        const int t0 = t_begin + j * TT;
        cp_async_tile<float2, KT>(sg[st], gb, t0, TT, p.L, k0, p.K, tid, KT);
        cp_async_flat<float>(sr[st], rb, (size_t)t0, TT, (size_t)p.L, tid, KT);
        cp_async_flat<float>(sp[st], pb, (size_t)t0, TT, (size_t)p.L, tid, KT);
        cp_async_commit();
    };
    if (ntiles > 0) issue(ntiles - 1, (ntiles - 1) & 1);
    for (int j = ntiles - 1; j >= 0; --j) {
        const int st = j & 1;
        if (j > 0) {
            issue(j - 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int t0 = t_begin + j * TT;
        const int rows = min(TT, t_end - t0);
        step_scalars(sr[st], sp[st], ssp, rows, tid);
        __syncthreads();
        for (int r0 = ((rows - 1) / CB) * CB; r0 >= 0; r0 -= CB) {
            float2 a[CB];
            transitions<CB>(a, lam * kLog2e, om, ssp, r0);
#pragma unroll
            for (int u = CB - 1; u >= 0; --u) {
                const int r = r0 + u;
                if (r < rows) {
                    const float2 gg = sg[st][r * KT + tid];
                    w = cmul_ca(a[u], make_float2(gg.x + w.x, gg.y + w.y));
                    P = cmul_ca(a[u], P);
                }
            }
        }
        __syncthreads();
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

// Producer side of the backward kernels: for the items i = 0..n-1 of the CTA's tile sequence
// (tile(i, t0, rows): the steps t0 .. t0+rows-1 of item i), the step scalars (softplus(r), phi)
// and the transitions a of the item's steps go into buffer i & 1, handed over with the FULL /
// EMPTY named barriers; the step scalars of item i + 1 are fetched while item i is computed.
template <typename TileFn>
__device__ __forceinline__ void cplx_produce(const CplxArgs& p, int n, TileFn tile, int tid, int k0,
                                             size_t boff, float2 (*sa)[FT * KT],
                                             float2 (*ssp)[FT]) {
    const int pt = tid - F_CONS, kk = pt % KT, rp = pt / KT;
    const int k = k0 + kk;
    const bool kv = k < p.K;
    const float lam2 = kv ? p.lam[k] * kLog2e : 0.0f, om = kv ? p.om[k] : 0.0f;
    const float* rb = p.r + boff;
    const float* pb = p.phi + boff;
    float rn = 0.0f, pn = 0.0f;
    if (n > 0 && pt < FT) {
        int t0, rows;
        tile(0, t0, rows);
        if (pt < rows) {
            rn = rb[t0 + pt];
            pn = pb[t0 + pt];
        }
    }
    for (int i = 0; i < n; ++i) {
        const int buf = i & 1;
        int t0, rows;
        tile(i, t0, rows);
        bar_sync_n(F_BAR_EMPTY + buf, F_NT);  // the consumers are done with buffer buf
        if (pt < FT) {
            ssp[buf][pt] = pt < rows ? make_float2(softplus_acc(rn), pn) : make_float2(0.0f, 0.0f);
            if (i + 1 < n) {
                int t1, r1;
                tile(i + 1, t1, r1);
                if (pt < r1) {
                    rn = rb[t1 + pt];
                    pn = pb[t1 + pt];
                }
            }
        }
        bar_sync_n(F_BAR_PROD, F_PROD);  // the step scalars are in
        float2 a[FT / 2];
        transitions_pk<FT / 2, 2>(a, lam2, om, ssp[buf], rp);
#pragma unroll
        for (int u = 0; u < FT / 2; ++u) sa[buf][(rp + 2 * u) * KT + kk] = a[u];
        bar_arrive_n(F_BAR_FULL + buf, F_NT);  // buffer buf holds the item's transitions
    }
    bar_sync_n(F_BAR_EMPTY + 0, F_NT);  // balance the consumers' last two releases
    bar_sync_n(F_BAR_EMPTY + 1, F_NT);
}

// Backward, warp-specialised like the forward: KT consumer threads (one per mode) sweep the
// adjoint backwards over 16-step tiles of g and h_{t-1} (their own two-stage cp.async ring) and
// sum (lambda Re q, omega Im q) over the CTA's modes per step; 2 KT producer threads compute the
// transitions of the next (earlier) tile, and the tile's step scalars (softplus(r), phi), into
// one of two shared buffers.
constexpr int B_USTAGES = 2;
constexpr int B_SMEM = ((2 + 2 * B_USTAGES) * FT * KT + 2 * FT) * (int)sizeof(float2);

__global__ void __launch_bounds__(F_NT) cplx_bwd_kernel(CplxArgs p) {
    static_assert(FT * 4 == KT, "column sums: four consumer threads per step");
    // dynamic shared memory (49.4 KB): transitions [2][FT*KT], g and h_{t-1} [B_USTAGES][FT*KT],
    // step scalars [2][FT].  The per-step (lambda Re q, omega Im q) overwrite the g of the tile
    // being swept: each consumer reads g at (r, mode) and then writes there, and the stage is not
    // refilled before the column sums that read them are done.
    extern __shared__ __align__(16) float2 cdyn[];
    float2 (*sa)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn);
    float2 (*sg)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn + 2 * FT * KT);
    float2 (*shp)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn + (2 + B_USTAGES) * FT * KT);
    float2 (*ssp)[FT] = reinterpret_cast<float2 (*)[FT]>(cdyn + (2 + 2 * B_USTAGES) * FT * KT);
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT;
    const int b = blockIdx.y, seg = blockIdx.z;
    const int t_begin = seg * p.seg_chunks * p.T;
    const int t_end = min(p.L, min(p.nC, (seg + 1) * p.seg_chunks) * p.T);
    const int ntiles = (t_end - t_begin + FT - 1) / FT;
    const size_t boff = (size_t)b * p.L;

    if (tid >= F_CONS) {
        // producers: the segment's tiles from the last one back
        cplx_produce(p, ntiles, [&](int i, int& t0, int& rows) {
            t0 = t_begin + (ntiles - 1 - i) * FT;
            rows = min(FT, t_end - t0);
        }, tid, k0, boff, sa, ssp);
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int k = k0 + tid;
    const bool kv = k < p.K;
    const float lam = kv ? p.lam[k] : 0.0f, om = kv ? p.om[k] : 0.0f;
    float2 w = make_float2(0.0f, 0.0f);
    if (seg < p.nseg - 1 && kv)
        w = reinterpret_cast<const float2*>(p.win)[((size_t)b * p.nseg + seg) * p.K + k];
    float dlam = 0.0f, dom = 0.0f;
    const float2* gb = reinterpret_cast<const float2*>(p.g) + boff * p.K;
    const float2* hb = reinterpret_cast<const float2*>(p.h_in) + boff * p.K;
    float2* dub = reinterpret_cast<float2*>(p.du) + boff * p.K;
    float2* partb = reinterpret_cast<float2*>(p.rp_part) + ((size_t)blockIdx.x * p.B + b) * (size_t)p.L;
    const int cs_r = tid >> 2, cs_part = tid & 3;  // column sums: step cs_r, a quarter of the modes
    auto issue = [&](int jt) {
        if (jt >= 0) {
            const int st = jt % B_USTAGES, t0 = t_begin + jt * FT;
            cp_async_tile<float2, KT>(sg[st], gb, t0, FT, p.L, k0, p.K, tid, F_CONS);
            if (t0 > 0) {
                cp_async_tile<float2, KT>(shp[st], hb, t0 - 1, FT, p.L, k0, p.K, tid, F_CONS);
            } else {  // h_{-1} = 0
                shp[st][tid] = make_float2(0.0f, 0.0f);
                cp_async_tile<float2, KT>(shp[st] + KT, hb, 0, FT - 1, p.L, k0, p.K, tid, F_CONS);
            }
        }
        cp_async_commit();
    };
    issue(ntiles - 1);
    bar_arrive_n(F_BAR_EMPTY + 0, F_NT);  // both transition buffers start empty
    bar_arrive_n(F_BAR_EMPTY + 1, F_NT);
    for (int i = 0; i < ntiles; ++i) {
        const int buf = i & 1, jt = ntiles - 1 - i, st = jt % B_USTAGES;
        const int t0 = t_begin + jt * FT, rows = min(FT, t_end - t0);
        cp_async_wait<0>();
        bar_sync_n(F_BAR_CONS, F_CONS);  // g, h of tile jt are in; both consumer warps are past jt+1
        issue(jt - 1);
        const float2* sgt = sg[st];
        const float2* sht = shp[st];
        const float2* sat = sa[buf];
        const float2* sst = ssp[buf];
        float2* red = sg[st];
        bar_sync_n(F_BAR_FULL + buf, F_NT);  // the producers have written the tile's transitions
#pragma unroll 4
        for (int r = rows - 1; r >= 0; --r) {
            const float2 sp2 = sst[r];
            const float2 av = sat[r * KT + tid];
            const float2 gg = sgt[r * KT + tid];
            const float2 mu = make_float2(gg.x + w.x, gg.y + w.y);
            w = cmul_ca(av, mu);
            const float2 q = cmul_cb(w, sht[r * KT + tid]);
            if (kv) dub[(size_t)(t0 + r) * p.K + k] = mu;
            dlam = fmaf(-sp2.x, q.x, dlam);
            dom = fmaf(sp2.y, q.y, dom);
            red[r * KT + tid] = make_float2(lam * q.x, om * q.y);
        }
        bar_arrive_n(F_BAR_EMPTY + buf, F_NT);  // transitions and step scalars are consumed
        bar_sync_n(F_BAR_CONS, F_CONS);         // the tile's (lambda Re q, omega Im q) are in
        {
            // sums over the CTA's modes, one step per four threads; the rotation by tid keeps
            // each half-warp's 8-byte loads in distinct banks
            float2 acc = make_float2(0.0f, 0.0f);
            const float2* row = red + cs_r * KT + cs_part * (KT / 4);
#pragma unroll
            for (int m = 0; m < KT / 4; ++m) {
                const float2 v = row[(m + tid) & (KT / 4 - 1)];
                acc.x += v.x;
                acc.y += v.y;
            }
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
            }
            if (cs_part == 0 && cs_r < rows) partb[t0 + cs_r] = acc;
        }
    }
    if (kv) {
        const size_t o = ((size_t)b * p.nseg + seg) * p.K + k;
        reinterpret_cast<float2*>(p.lo_part)[o] = make_float2(dlam, dom);
        if (!(isfinite(w.x) && isfinite(w.y))) flag_status(p.status, kStatusNonFinite);
    }
}

// Checkpointed backward: the same adjoint sweep, with the trajectory recomputed chunk by chunk
// from the forward's checkpoints instead of read from a stored h ("Breaking the Memory Wall ...
// Tiled Operator-Space Evolution", abstract: only chunk-boundary states are kept).  For each chunk
// of the segment, last first, the CTA's tile sequence holds the chunk's tiles twice: forward, where
// the consumers run h = a h + u from the chunk's entering checkpoint and leave h_{t-1} of every step
// in the CTA's scratch region ([T][KT] complex, L2-resident), then backward, where they sweep the
// adjoint exactly as cplx_bwd_kernel does with h_{t-1} read back from that region.  The producers
// compute the transitions of every item, so each transition is evaluated twice.
__global__ void __launch_bounds__(F_NT) cplx_bwd_ckpt_kernel(CplxArgs p) {
    static_assert(FT * 4 == KT, "column sums: four consumer threads per step");
    // dynamic shared memory as cplx_bwd_kernel: transitions [2][FT*KT], u (forward items) or g
    // (sweep items) [B_USTAGES][FT*KT], h_{t-1} [B_USTAGES][FT*KT], step scalars [2][FT]
    extern __shared__ __align__(16) float2 cdyn[];
    float2 (*sa)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn);
    float2 (*sx)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn + 2 * FT * KT);
    float2 (*shp)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn + (2 + B_USTAGES) * FT * KT);
    float2 (*ssp)[FT] = reinterpret_cast<float2 (*)[FT]>(cdyn + (2 + 2 * B_USTAGES) * FT * KT);
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT;
    const int b = blockIdx.y, seg = p.seg0 + blockIdx.z;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);
    const int ntT = p.T / FT;                                   // tiles of a full chunk
    const int nt0 = (min(p.T, p.L - (c_end - 1) * p.T) + FT - 1) / FT;  // of the segment's last
    const int n = c_end > c_begin ? 2 * nt0 + 2 * ntT * (c_end - 1 - c_begin) : 0;
    const size_t boff = (size_t)b * p.L;
    // item i: chunk c, forward (sweep = false) or sweep item, tile j of the chunk's nt tiles
    auto item = [&](int i, int& c, bool& sweep, int& j, int& nt) {
        if (i < 2 * nt0) {
            c = c_end - 1;
            nt = nt0;
            j = i;
        } else {
            const int i2 = i - 2 * nt0;
            c = c_end - 2 - i2 / (2 * ntT);
            nt = ntT;
            j = i2 % (2 * ntT);
        }
        sweep = j >= nt;
        if (sweep) j = 2 * nt - 1 - j;
    };

    if (tid >= F_CONS) {
        cplx_produce(p, n, [&](int i, int& t0, int& rows) {
            int c, j, nt;
            bool sw;
            item(i, c, sw, j, nt);
            t0 = c * p.T + j * FT;
            rows = min(FT, p.L - t0);
        }, tid, k0, boff, sa, ssp);
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int k = k0 + tid;
    const bool kv = k < p.K;
    const float lam = kv ? p.lam[k] : 0.0f, om = kv ? p.om[k] : 0.0f;
    float2 w = make_float2(0.0f, 0.0f), h = make_float2(0.0f, 0.0f);
    if (seg < p.nseg - 1 && kv)
        w = reinterpret_cast<const float2*>(p.win)[((size_t)b * p.nseg + seg) * p.K + k];
    float dlam = 0.0f, dom = 0.0f;
    const float2* ub = reinterpret_cast<const float2*>(p.u) + boff * p.K;
    const float2* gb = reinterpret_cast<const float2*>(p.g) + boff * p.K;
    const float2* ckb = reinterpret_cast<const float2*>(p.ckpt_in) + (size_t)b * p.nC * p.K;
    float2* dub = reinterpret_cast<float2*>(p.du) + boff * p.K;
    float2* partb = reinterpret_cast<float2*>(p.rp_part) + ((size_t)blockIdx.x * p.B + b) * (size_t)p.L;
    const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    float2* traj = reinterpret_cast<float2*>(p.traj) + cta * (cplx_traj_floats(p.T) / 2);
    const int cs_r = tid >> 2, cs_part = tid & 3;  // column sums: step cs_r, a quarter of the modes
    // copies of item i: part 1 = its u or g tile, part 2 = its h_{t-1} rows (sweep items); both
    // parts by default
    auto issue = [&](int i, int parts = 3) {
        if (i < n) {
            int c, j, nt;
            bool sw;
            item(i, c, sw, j, nt);
            const int st = i % B_USTAGES, t0 = c * p.T + j * FT;
            if (parts & 1) cp_async_tile<float2, KT>(sx[st], sw ? gb : ub, t0, FT, p.L, k0, p.K, tid, F_CONS);
            if (sw && (parts & 2))
                cp_async_tile<float2, KT>(shp[st], traj, j * FT, FT, min(p.T, p.L - c * p.T), 0,
                                          KT, tid, F_CONS);
        }
        cp_async_commit();
    };
    issue(0);
    bar_arrive_n(F_BAR_EMPTY + 0, F_NT);  // both transition buffers start empty
    bar_arrive_n(F_BAR_EMPTY + 1, F_NT);
    for (int i = 0; i < n; ++i) {
        int c, j, nt;
        bool sweep;
        item(i, c, sweep, j, nt);
        const int buf = i & 1, st = i % B_USTAGES;
        const int t0 = c * p.T + j * FT, rows = min(FT, p.L - t0);
        cp_async_wait<0>();
        bar_sync_n(F_BAR_CONS, F_CONS);  // item i's tiles are in; every consumer is past item i-1
        // the first sweep item of a chunk reads the h_{t-1} that the item before it writes, so
        // those rows are copied once that item is done (its g tile right away)
        const bool defer = !sweep && j == nt - 1;
        issue(i + 1, defer ? 1 : 3);
        const float2* sat = sa[buf];
        bar_sync_n(F_BAR_FULL + buf, F_NT);  // the producers have written the item's transitions
        if (!sweep) {
            if (j == 0 && kv) h = c > 0 ? ckb[(size_t)(c - 1) * p.K + k] : make_float2(0.0f, 0.0f);
            const float2* sut = sx[st];
            float2* tr = traj + (size_t)(j * FT) * KT + tid;
#pragma unroll 4
            for (int r = 0; r < rows; ++r) {
                tr[r * KT] = h;  // h_{t-1} of step t = t0 + r
                const float2 ah = cmul(sat[r * KT + tid], h);
                const float2 uu = sut[r * KT + tid];
                h = make_float2(ah.x + uu.x, ah.y + uu.y);
            }
            bar_arrive_n(F_BAR_EMPTY + buf, F_NT);  // transitions consumed
            if (defer) {
                bar_sync_n(F_BAR_CONS, F_CONS);  // the chunk's h_{t-1} are all written
                issue(i + 1, 2);
            }
            continue;
        }
        const float2* sgt = sx[st];
        const float2* sht = shp[st];
        const float2* sst = ssp[buf];
        float2* red = sx[st];
#pragma unroll 4
        for (int r = rows - 1; r >= 0; --r) {
            const float2 sp2 = sst[r];
            const float2 av = sat[r * KT + tid];
            const float2 gg = sgt[r * KT + tid];
            const float2 mu = make_float2(gg.x + w.x, gg.y + w.y);
            w = cmul_ca(av, mu);
            const float2 q = cmul_cb(w, sht[r * KT + tid]);
            if (kv) dub[(size_t)(t0 + r) * p.K + k] = mu;
            dlam = fmaf(-sp2.x, q.x, dlam);
            dom = fmaf(sp2.y, q.y, dom);
            red[r * KT + tid] = make_float2(lam * q.x, om * q.y);
        }
        bar_arrive_n(F_BAR_EMPTY + buf, F_NT);  // transitions and step scalars are consumed
        bar_sync_n(F_BAR_CONS, F_CONS);         // the item's (lambda Re q, omega Im q) are in
        {
            float2 acc = make_float2(0.0f, 0.0f);
            const float2* row = red + cs_r * KT + cs_part * (KT / 4);
#pragma unroll
            for (int m = 0; m < KT / 4; ++m) {
                const float2 v = row[(m + tid) & (KT / 4 - 1)];
                acc.x += v.x;
                acc.y += v.y;
            }
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
            }
            if (cs_part == 0 && cs_r < rows) partb[t0 + cs_r] = acc;
        }
    }
    if (kv) {
        const size_t o = ((size_t)b * p.nseg + seg) * p.K + k;
        reinterpret_cast<float2*>(p.lo_part)[o] = make_float2(dlam, dom);
        if (!(isfinite(w.x) && isfinite(w.y))) flag_status(p.status, kStatusNonFinite);
    }
}

// Exact structured RTRL (SPARC abstract: exact structured real-time recurrent learning for online
// credit assignment).  The state's forward-mode sensitivities to the mode's own lambda and omega
// travel with it,
//   S^lambda_t = a_t S^lambda_{t-1} - s_t a_t h_{t-1},   S^omega_t = a_t S^omega_{t-1} + i phi_t a_t h_{t-1},
// and the gradient of Re sum conj(g) h accumulates as the steps arrive:
//   dlambda += Re(conj(g_t) S^lambda_t),  domega += Re(conj(g_t) S^omega_t).
// One forward pass, no reverse sweep, nothing of the trajectory kept (h is written only if asked).
// A CTA takes KT modes of one batch row over the whole sequence.
__global__ void __launch_bounds__(F_NT) cplx_rtrl_kernel(CplxArgs p) {
    // warp-specialised like the forward: KT consumer threads carry (h, S^lambda, S^omega) of one
    // mode each over 16-step tiles of u and g (their own two-stage cp.async ring); 2 KT producer
    // threads compute the next tile's transitions and step scalars into one of two buffers.
    // Dynamic shared memory (49.4 KB): transitions [2][FT*KT], u and g [B_USTAGES][FT*KT], step
    // scalars [2][FT].
    extern __shared__ __align__(16) float2 cdyn[];
    float2 (*sa)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn);
    float2 (*su)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn + 2 * FT * KT);
    float2 (*sgt)[FT * KT] = reinterpret_cast<float2 (*)[FT * KT]>(cdyn + (2 + B_USTAGES) * FT * KT);
    float2 (*ssp)[FT] = reinterpret_cast<float2 (*)[FT]>(cdyn + (2 + 2 * B_USTAGES) * FT * KT);
    const int tid = threadIdx.x;
    const int k0 = blockIdx.x * KT;
    const int b = blockIdx.y;
    const int ntiles = (p.L + FT - 1) / FT;
    const size_t boff = (size_t)b * p.L;

    if (tid >= F_CONS) {
        // ---------------------------------------------------------------- producers
        const int pt = tid - F_CONS, kk = pt % KT, rp = pt / KT;
        const int k = k0 + kk;
        const bool kv = k < p.K;
        const float lam2 = kv ? p.lam[k] * kLog2e : 0.0f, om = kv ? p.om[k] : 0.0f;
        const float* rb = p.r + boff;
        const float* pb = p.phi + boff;
        float rn = 0.0f, pn = 0.0f;  // step scalars of the next tile, fetched a tile ahead
        if (pt < FT && pt < p.L) {
            rn = rb[pt];
            pn = pb[pt];
        }
        for (int i = 0; i < ntiles; ++i) {
            const int buf = i & 1;
            const int t0 = i * FT, rows = min(FT, p.L - t0);
            bar_sync_n(F_BAR_EMPTY + buf, F_NT);  // the consumers are done with buffer buf
            if (pt < FT) {
                ssp[buf][pt] = pt < rows ? make_float2(softplus_acc(rn), pn) : make_float2(0.0f, 0.0f);
                const int tn = t0 + FT + pt;
                if (tn < p.L) {
                    rn = rb[tn];
                    pn = pb[tn];
                }
            }
            bar_sync_n(F_BAR_PROD, F_PROD);  // the step scalars are in
            float2 a[FT / 2];
            transitions_pk<FT / 2, 2>(a, lam2, om, ssp[buf], rp);
#pragma unroll
            for (int u = 0; u < FT / 2; ++u) sa[buf][(rp + 2 * u) * KT + kk] = a[u];
            bar_arrive_n(F_BAR_FULL + buf, F_NT);
        }
        bar_sync_n(F_BAR_EMPTY + 0, F_NT);  // balance the consumers' last two releases
        bar_sync_n(F_BAR_EMPTY + 1, F_NT);
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int k = k0 + tid;
    const bool kv = k < p.K;
    float2* stb = p.state ? reinterpret_cast<float2*>(p.state) + (size_t)b * 3 * p.K : nullptr;
    float2 h = make_float2(0.0f, 0.0f), Sl = h, So = h;
    if (stb && kv) {
        h = stb[k];
        Sl = stb[p.K + k];
        So = stb[2 * p.K + k];
    }
    float dl = 0.0f, dom = 0.0f;
    const float2* ub = reinterpret_cast<const float2*>(p.u) + boff * p.K;
    const float2* gb = reinterpret_cast<const float2*>(p.g) + boff * p.K;
    float2* hb = p.h ? reinterpret_cast<float2*>(p.h) + boff * p.K : nullptr;
    auto issue = [&](int i) {
        if (i < ntiles) {
            const int st = i % B_USTAGES;
            cp_async_tile<float2, KT>(su[st], ub, i * FT, FT, p.L, k0, p.K, tid, F_CONS);
            cp_async_tile<float2, KT>(sgt[st], gb, i * FT, FT, p.L, k0, p.K, tid, F_CONS);
        }
        cp_async_commit();
    };
    issue(0);
    bar_arrive_n(F_BAR_EMPTY + 0, F_NT);  // both transition buffers start empty
    bar_arrive_n(F_BAR_EMPTY + 1, F_NT);
    for (int i = 0; i < ntiles; ++i) {
        const int buf = i & 1, st = i % B_USTAGES;
        const int t0 = i * FT, rows = min(FT, p.L - t0);
        cp_async_wait<0>();
        bar_sync_n(F_BAR_CONS, F_CONS);  // u, g of tile i are in; both consumer warps are past i-1
        issue(i + 1);
        const float2* sut = su[st];
        const float2* sgg = sgt[st];
        const float2* sat = sa[buf];
        const float2* sst = ssp[buf];
        bar_sync_n(F_BAR_FULL + buf, F_NT);  // the producers have written the tile's transitions
#pragma unroll 4
        for (int r = 0; r < rows; ++r) {
            const float2 sp2 = sst[r];  // (s, phi)
            const float2 av = sat[r * KT + tid];
            const float2 ah = cmul(av, h);
            const float2 al = cmul(av, Sl), ao = cmul(av, So);
            Sl = make_float2(fmaf(-sp2.x, ah.x, al.x), fmaf(-sp2.x, ah.y, al.y));
            So = make_float2(fmaf(-sp2.y, ah.y, ao.x), fmaf(sp2.y, ah.x, ao.y));
            const float2 uu = sut[r * KT + tid];
            h = make_float2(ah.x + uu.x, ah.y + uu.y);
            const float2 gg = sgg[r * KT + tid];
            dl = fmaf(gg.x, Sl.x, fmaf(gg.y, Sl.y, dl));
            dom = fmaf(gg.x, So.x, fmaf(gg.y, So.y, dom));
            if (hb && kv) hb[(size_t)(t0 + r) * p.K + k] = h;
        }
        bar_arrive_n(F_BAR_EMPTY + buf, F_NT);
    }
    if (kv) {
        reinterpret_cast<float2*>(p.lo_part)[(size_t)b * p.K + k] = make_float2(dl, dom);
        if (stb) {
            stb[k] = h;
            stb[p.K + k] = Sl;
            stb[2 * p.K + k] = So;
        }
        if (!(isfinite(h.x) && isfinite(h.y) && isfinite(Sl.x) && isfinite(Sl.y) &&
              isfinite(So.x) && isfinite(So.y)))
            flag_status(p.status, kStatusNonFinite);
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
        cplx_fwd_kernel<true><<<dim3(a.nkt, a.B, a.nseg - 1), F_NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.K;
        cplx_carry_fwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            a.B, a.nseg, a.K, reinterpret_cast<const float2*>(a.sumP),
            reinterpret_cast<const float2*>(a.sumS), reinterpret_cast<float2*>(a.hin));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cplx_fwd_kernel<false><<<dim3(a.nkt, a.B, a.nseg), F_NT, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_cplx_rtrl(const CplxArgs& a, cudaStream_t st) {
    cudaError_t e;
    e = cudaFuncSetAttribute(cplx_rtrl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM);
    if (e != cudaSuccess) return e;
    cplx_rtrl_kernel<<<dim3(a.nkt, a.B, 1), F_NT, B_SMEM, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cplx_reduce_k_kernel<<<(a.K + 255) / 256, 256, 0, st>>>(a);  // sums over b (nseg = 1)
    return cudaGetLastError();
}

cudaError_t launch_cplx_bwd_ckpt(const CplxArgs& a0, int group, cudaStream_t st) {
    cudaError_t e;
    CplxArgs a = a0;
    if (a.nseg > 1) {
        cplx_bwd_summary_kernel<<<dim3(a.nkt, a.B, a.nseg - 1), KT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.K;
        cplx_carry_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            a.B, a.nseg, a.K, reinterpret_cast<const float2*>(a.gsumP),
            reinterpret_cast<const float2*>(a.gsumG), reinterpret_cast<float2*>(a.win));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(cplx_bwd_ckpt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM);
    if (e != cudaSuccess) return e;
    for (int lo = 0; lo < a.nseg; lo += group) {
        a.seg0 = lo;
        const int ns = a.nseg - lo < group ? a.nseg - lo : group;
        cplx_bwd_ckpt_kernel<<<dim3(a.nkt, a.B, ns), F_NT, B_SMEM, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int64_t n = (int64_t)a.B * a.L;
    if (n > 0) {
        cplx_reduce_bl_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cplx_reduce_k_kernel<<<(a.K + 255) / 256, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_cplx_bwd(const CplxArgs& a, cudaStream_t st) {
    cudaError_t e;
    if (a.nseg > 1) {
        cplx_bwd_summary_kernel<<<dim3(a.nkt, a.B, a.nseg - 1), KT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.K;
        cplx_carry_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            a.B, a.nseg, a.K, reinterpret_cast<const float2*>(a.gsumP),
            reinterpret_cast<const float2*>(a.gsumG), reinterpret_cast<float2*>(a.win));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(cplx_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM);
    if (e != cudaSuccess) return e;
    cplx_bwd_kernel<<<dim3(a.nkt, a.B, a.nseg), F_NT, B_SMEM, st>>>(a);
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
