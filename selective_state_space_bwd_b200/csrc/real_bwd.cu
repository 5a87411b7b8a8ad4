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
// segment, v <- a_t (C_t dy_t + v), and P = prod a over the segment.  The segment streams through
// shared memory from its end backwards in 32-step sub-tiles of dy, delta_raw and C, copied
// asynchronously two sub-tiles ahead (three-stage ring), so the copies' latency stays off the
// scan.
template <typename E, int N>
struct BwdSumSmem {
    static constexpr int TS = 32, DT = kRealDT;
    static constexpr int XE = TS * DT, CE = TS * N;
    static constexpr int RAW = 3;                                      // raw stages
    static constexpr int STAGE = (2 * XE + CE) * (int)sizeof(E);       // dy, delta_raw, C as stored
    static constexpr int DEL = RAW * STAGE;                            // delta [TS][DT] fp32
    static constexpr int CF = DEL + XE * 4;                            // C [TS][N] fp32
    static constexpr int BYTES = CF + CE * 4;
};

template <typename E, int N, int S>
__global__ void __launch_bounds__(RealCfg<N, S>::NT) real_bwd_summary_kernel(RealArgs p) {
    using Cfg = RealCfg<N, S>;
    using Sm = BwdSumSmem<E, N>;
    constexpr int P2 = Cfg::P2, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT, U = Cfg::U, TS = Sm::TS;
    extern __shared__ __align__(16) unsigned char smem[];
    float* sdel = reinterpret_cast<float*>(smem + Sm::DEL);
    float* sCf = reinterpret_cast<float*>(smem + Sm::CF);

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int b = blockIdx.y, seg = blockIdx.z + 1;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * S;
    const bool dv = d < p.D;
    const int t_begin = seg * p.seg_chunks * p.T;
    const int t_end = min(p.L, min(p.nC, (seg + 1) * p.seg_chunks) * p.T);
    const int nsub = t_end > t_begin ? (t_end - t_begin + TS - 1) / TS : 0;

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

    auto raw = [&](int k) { return reinterpret_cast<E*>(smem + (k % Sm::RAW) * Sm::STAGE); };
    // sub-tile k holds steps [t_begin + k TS, min(t_end, t_begin + (k + 1) TS)), rounded up to
    // whole groups of U; the rounding only reaches past the sequence end (segment ends are
    // multiples of the chunk length), where the copies read zeros
    auto issue = [&](int k) {
        if (k >= 0) {
            const int t0 = t_begin + k * TS;
            const int rows4 = (min(TS, t_end - t0) + U - 1) / U * U;
            E* sr = raw(k);
            cp_async_tile<E, DT>(sr, dyb, t0, rows4, p.L, d0, p.D, tid, NT);
            cp_async_tile<E, DT>(sr + Sm::XE, drb, t0, rows4, p.L, d0, p.D, tid, NT);
            cp_async_flat<E>(sr + 2 * Sm::XE, Cb, (size_t)t0 * N, rows4 * N, (size_t)p.L * N, tid, NT);
        }
        cp_async_commit();  // an empty group before the first sub-tile keeps the wait counts uniform
    };
    issue(nsub - 1);
    issue(nsub - 2);
    for (int k = nsub - 1; k >= 0; --k) {
        cp_async_wait<1>();  // sub-tile k is in (k - 1 may still be in flight)
        __syncthreads();     // ... for every thread, and every thread is past the scan of k + 1
        issue(k - 2);
        const int t0 = t_begin + k * TS;
        const int rows = min(TS, t_end - t0);
        const int rows4 = (rows + U - 1) / U * U;
        const E* sdy = raw(k);
        const E* sdr = sdy + Sm::XE;
        const E* sC = sdy + 2 * Sm::XE;
        // steps past the sequence end get delta = 0 (a = 1; their dy reads zero)
        for (int i = tid; i < rows4 * DT; i += NT)
            sdel[i] = i < rows * DT ? softplus_fast(Elem<E>::to_f(sdr[i])) : 0.0f;
        for (int i = tid; i < rows4 * N; i += NT) sCf[i] = Elem<E>::to_f(sC[i]);
        __syncthreads();
        for (int r0 = rows4 - U; r0 >= 0; r0 -= U) {
#pragma unroll
            for (int u = U - 1; u >= 0; --u) {
                const int r = r0 + u;
                const float dlt = sdel[r * DT + dl];
                const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                float2 cq[P2];
                ld_pairs<S>(cq, sCf + r * N + n0);
#pragma unroll
                for (int i = 0; i < P2; ++i) {
                    const float2 a = ex2_pair(__fmul2_rn(f2(dlt), A2[i]));
                    v[i] = __fmul2_rn(a, __ffma2_rn(cq[i], f2(dyv), v[i]));
                    P[i] = __fmul2_rn(P[i], a);
                }
            }
        }
    }
    cp_async_wait<0>();  // no copy outlives the CTA
    if (dv) {
        const size_t o = (((size_t)b * (p.nseg - 1) + (seg - 1)) * p.D + d) * N + n0;
        st_pairs<S>(p.gsumP + o, P);
        st_pairs<S>(p.gsumG + o, v);
    }
}

// Scaled adjoint entering each segment from its end: v_in[nseg-1] = dhL (or 0, read by the last
// segment directly), v_in[s-1] = G_s + P_s v_in[s].  v_in[s-1] overwrites G_s in place (slot s-1
// of the summaries), so the hand-over needs no buffer of its own.
__global__ void real_carry_bwd_kernel(int B, int nseg, int DN, const float* __restrict__ P,
                                      float* __restrict__ G, const float* __restrict__ dhL) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * DN) return;
    const int b = (int)(i / DN), k = (int)(i % DN);
    float v = dhL ? dhL[i] : 0.0f;
    for (int s = nseg - 1; s > 0; --s) {
        const size_t j = ((size_t)b * (nseg - 1) + (s - 1)) * DN + k;
        v = fmaf(P[j], v, G[j]);
        G[j] = v;
    }
}

// ------------------------------------------------------------------------------------------------
// Backward main kernel.  Chunks of the segment in reverse order; per chunk:
//   pass A: stream the chunk forward in 32-step sub-tiles (asynchronous two-stage ring).  Per
//           sub-tile: delta and sigmoid(delta_raw) from one exp per (t, d); (delta, sigma) and
//           the state at every 4-step window start go to this CTA's L2-resident workspace region;
//           the recurrence advances through the sub-tile.
//   pass B: stream the sub-tiles in reverse.  For each 4-step window, last first: recompute
//           (a_t, a_t h_{t-1}) forward from the window's start state into registers, then sweep
//           the adjoint back through the window.
// Channel sums of dB and dC.  A thread's four state slots are rotated by its position `rot` among
// four neighbouring channel lanes (slot j holds state n0 + ((j + rot) & 3)), so after each step
// the four lanes exchange their per-slot values in three shuffle rounds that all send the same
// slot (an all-to-all with uniform register indices): each lane ends with the sum over the four
// channels of one state, for dB and for dC.  After each window the eight four-channel groups of
// the CTA meet in shared memory and one thread per (step, dB or dC, state) adds them into the
// CTA's partial row.  The per-(t, d) sums over the states (dx, ddelta_raw) are a reduce-scatter
// over the NG lanes of a channel, per window.
template <int N>
struct BwdCfg {
    static constexpr int S = 4;            // states per thread
    static constexpr int P2 = 2;           // state pairs per thread
    static constexpr int NG = N / S;       // lanes per channel
    static constexpr int DT = kRealDT;     // channels per CTA
    static constexpr int NT = DT * NG;     // threads per CTA
    static constexpr int W = 4;            // steps per window
    static constexpr int TT = 32;          // steps per staged sub-tile
    static constexpr int GRP = DT / 4;     // four-channel groups per CTA
    static constexpr int RS = 9 * N;       // stride (floats) of a group's window sums in shared memory
    static_assert(W * 2 * N == NT, "one (step, dB or dC, state) output of a window per thread");
};

// A2A selects the channel sums of dB / dC: the four-lane all-to-all over rotated slots (fewer
// instructions; B and C are staged in their four rotations and the CTA adds eight group partials
// per output) or a shuffle reduce-scatter over the warp's eight channels with natural slot order
// (plain B / C tiles, four warp partials per output), which needs fewer registers and less shared
// memory and is used by the instance compiled for four CTAs per SM.
template <typename E, int N, bool A2A>
struct BwdSmem {
    using Cfg = BwdCfg<N>;
    static constexpr int TT = Cfg::TT, DT = Cfg::DT;
    static constexpr int XE = TT * DT, BE = TT * N;
    static constexpr int ROT = A2A ? 4 : 1;  // slot rotations staged per B / C row
    static constexpr int RE = TT * ROT * N;  // fp32 tile of B or C
    // pass A stage: x, delta_raw, B (raw)
    static constexpr int A_STAGE = (2 * XE + BE) * (int)sizeof(E);
    static constexpr int A_DD = 2 * A_STAGE;              // (delta, delta*x) float2 [TT][DT]
    static constexpr int A_BR = A_DD + XE * 8;            // B rotated fp32 [TT][4][N]
    static constexpr int A_END = A_BR + RE * 4;
    // pass B stage: (delta, sigma) float2, x, dy, B, C (raw)
    static constexpr int B_STAGE = XE * 8 + (2 * XE + 2 * BE) * (int)sizeof(E);
    static constexpr int B_BR = 2 * B_STAGE;              // B rotated fp32
    static constexpr int B_CR = B_BR + RE * 4;            // C rotated fp32
    static constexpr int B_RED = B_CR + RE * 4;           // window sums, double-buffered
    static constexpr int RED = A2A ? Cfg::GRP * Cfg::RS : (Cfg::NT / 32) * 2 * N * Cfg::W;
    static constexpr int B_END = B_RED + 2 * RED * 4;
    static constexpr int BYTES = A_END > B_END ? A_END : B_END;
    static_assert(A_STAGE % 16 == 0 && B_STAGE % 16 == 0, "16-byte aligned stages");
};

// Rows [0, rows) of a staged [rows][N] tile to fp32 with the four slot rotations of every group of
// four states: dst[(row * 4 + k) * N + 4 g + j] = src[row * N + 4 g + ((j + k) & 3)], so a thread
// of rotation k reads its four slots with one 16-byte load.
template <typename E, int N, int ROT>
__device__ __forceinline__ void rotate_rows(float* __restrict__ dst, const E* __restrict__ src,
                                            int rows, int tid, int nthreads) {
    constexpr int G = N / 4;
    for (int i = tid; i < rows * G; i += nthreads) {
        const int row = i / G, g = i - row * G;
        float v[4];
        if constexpr (sizeof(E) == 2) {
            const uint2 w = *reinterpret_cast<const uint2*>(src + row * N + 4 * g);
            v[0] = __uint_as_float(w.x << 16);
            v[1] = __uint_as_float(w.x & 0xffff0000u);
            v[2] = __uint_as_float(w.y << 16);
            v[3] = __uint_as_float(w.y & 0xffff0000u);
        } else {
            const float4 w = *reinterpret_cast<const float4*>(src + row * N + 4 * g);
            v[0] = w.x;
            v[1] = w.y;
            v[2] = w.z;
            v[3] = w.w;
        }
        float* o = dst + row * ROT * N + 4 * g;
#pragma unroll
        for (int k = 0; k < ROT; ++k)
            *reinterpret_cast<float4*>(o + k * N) =
                make_float4(v[k & 3], v[(k + 1) & 3], v[(k + 2) & 3], v[(k + 3) & 3]);
    }
}

// The thread's four slots of one state row (a [.., N] row of a [*, D, N] array), in slot order.
__device__ __forceinline__ void ld_slots(float2 (&o)[2], const float* row, const int (&sidx)[4]) {
    o[0] = make_float2(row[sidx[0]], row[sidx[1]]);
    o[1] = make_float2(row[sidx[2]], row[sidx[3]]);
}
__device__ __forceinline__ void st_slots(float* row, const float2 (&o)[2], const int (&sidx)[4]) {
    row[sidx[0]] = o[0].x;
    row[sidx[1]] = o[0].y;
    row[sidx[2]] = o[1].x;
    row[sidx[3]] = o[1].y;
}

// A scratch slot for this CTA: claims a clear bit of the slot mask (the search starts at `start`),
// or returns -1 once the bounded wait gives up.  A slot is held from a CTA's start to its end, so
// with at least as many slots as resident CTAs a clear bit exists whenever a CTA starts; with
// fewer, a CTA waits for a holder to finish (holders never wait), which the bound allows for.
constexpr unsigned kSlotSpinLimit = 1u << 22;  // x 256 ns sleeps: about a second
__device__ int claim_slot(unsigned* mask, int nslot, int start) {
    // first the CTA's own slot (CTAs of a launch with no more CTAs than slots never meet)
    {
        const unsigned bit = 1u << (start & 31);
        if (!(atomicOr(mask + start / 32, bit) & bit)) {
            __threadfence();
            return start;
        }
    }
    const int nw = (nslot + 31) / 32;
    for (unsigned it = 0; it < kSlotSpinLimit; ++it) {
        for (int k = 0; k < nw; ++k) {
            const int w = (start / 32 + k) % nw;
            const unsigned valid = (w == nw - 1 && (nslot & 31)) ? (1u << (nslot & 31)) - 1u : ~0u;
            unsigned clear = ~*reinterpret_cast<volatile unsigned*>(mask + w) & valid;
            while (clear) {
                const unsigned bit = 1u << (__ffs(clear) - 1);
                const unsigned old = atomicOr(mask + w, bit);
                if (!(old & bit)) {
                    __threadfence();  // the previous holder's accesses come first
                    return w * 32 + (__ffs(bit) - 1);
                }
                clear = ~old & valid;
            }
        }
        __nanosleep(256);
    }
    return -1;
}

// MINB: CTAs per SM the register allocation must allow.  4 (126 registers for the Euler N = 16
// kernel) lets grids of up to 592 CTAs run in one wave; 3 leaves the compiler more registers,
// which is faster when the grid fits 3 per SM anyway (zero-order hold always uses 3).
// Fused dB/dC sums (FUSED, launches whose CTAs are all resident: cooperative launches).  The
// CTAs of one (segment, batch row) walk the same chunks in the same order.  After a chunk's pass B
// a CTA counts itself finished with that chunk; after the next chunk's pass A (or at its end) it
// waits until all ndt CTAs of its row have finished the chunk, then sums its share of the
// chunk's partial rows (rows [rows * dt / ndt, rows * (dt + 1) / ndt)) over the channel tiles
// into dB / dC: the share's float4 units times P parts of the tiles spread over the threads (about
// eight tiles each, their loads issued together), the parts added in part order.  With N = 16 a
// partial row is one 128-byte line; those lines are then dead and are discarded from L2, so that
// they are never written back.  Kept out of line: the scan kernel's registers stay its own.
template <typename E, int N>
__device__ __noinline__ void fused_dbc_share(const float* __restrict__ part, int part_rows, int part_t0,
                                             int B, int L, int T, int ndt, E* __restrict__ dB,
                                             E* __restrict__ dC, int b, int chunk, int dt, int tid,
                                             int nthreads, float4* comb) {
    constexpr int N2 = 2 * N, U4 = N2 / 4;            // float4 columns of a partial row
    const int t0 = chunk * T;
    const int rows = min(T, L - t0);
    const int r0 = (int)((int64_t)rows * dt / ndt), r1 = (int)((int64_t)rows * (dt + 1) / ndt);
    const int U = (r1 - r0) * U4;                      // float4 units of the share
    const size_t stride = (size_t)B * part_rows * N2;  // between channel tiles' partials
    const float* base = part + ((size_t)b * part_rows + (t0 - part_t0) + r0) * N2;
    for (int ub = 0; ub < U; ub += nthreads) {
        const int nu = min(nthreads, U - ub);
        const int P = nthreads / nu;                   // parts of the tiles
        const int tp = (ndt + P - 1) / P;
        const int unit = tid % nu, pq = tid / nu;
        const int u = ub + unit;
        if (pq < P) {
            float4 s = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            const float* src = base + (size_t)(u / U4) * N2 + (u % U4) * 4;
            const int j0 = min(ndt, pq * tp), j1 = min(ndt, j0 + tp);
            int j = j0;
            for (; j + 8 <= j1; j += 8) {
                float4 v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = __ldcg(reinterpret_cast<const float4*>(src + (size_t)(j + k) * stride));
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    s.x += v[k].x;
                    s.y += v[k].y;
                    s.z += v[k].z;
                    s.w += v[k].w;
                }
            }
            for (; j < j1; ++j) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (size_t)j * stride));
                s.x += v.x;
                s.y += v.y;
                s.z += v.z;
                s.w += v.w;
            }
            comb[pq * nu + unit] = s;
        }
        __syncthreads();
        if (pq == 0) {
            float4 t = comb[unit];
            for (int w = 1; w < P; ++w) {
                const float4 v = comb[w * nu + unit];
                t.x += v.x;
                t.y += v.y;
                t.z += v.z;
                t.w += v.w;
            }
            const float o[4] = {t.x, t.y, t.z, t.w};
            const int r = r0 + u / U4, e = (u % U4) * 4;
            const size_t bl = (size_t)b * L + t0 + r;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (e + k < N)
                    dB[bl * N + e + k] = Elem<E>::from_f(o[k]);
                else
                    dC[bl * N + (e + k - N)] = Elem<E>::from_f(o[k]);
            }
        }
        __syncthreads();
    }
    if constexpr (N2 * 4 == 128) {
        // every tile's partial rows of the share, one line each, are dead: drop them unwritten
        for (int i = tid; i < (r1 - r0) * ndt; i += nthreads) {
            const int jt = i / (r1 - r0), r = i % (r1 - r0);
            const float* a = base + (size_t)jt * stride + (size_t)r * N2;
            asm volatile("discard.global.L2 [%0], 128;\n" ::"l"(a) : "memory");
        }
    }
}

template <typename E, int N, bool ZOH, int MINB, bool A2A, bool POOL, bool FUSED>
__global__ void __launch_bounds__(BwdCfg<N>::NT, MINB) real_bwd_kernel(RealArgs p) {
    using Cfg = BwdCfg<N>;
    using Sm = BwdSmem<E, N, A2A>;
    constexpr int ROT = Sm::ROT;
    constexpr int P2 = Cfg::P2, NG = Cfg::NG, DT = Cfg::DT, NT = Cfg::NT, W = Cfg::W;
    constexpr int GRP = Cfg::GRP, RS = Cfg::RS;
    // per-step channel sums over the states: sum g w' B (dx), sum A q, and for zero-order hold
    // also sum g a B (ddelta; with Euler it equals the first)
    constexpr int SV = ZOH ? 3 : 2;
    // zero-order hold: E1 of a window's steps kept in registers from the recompute, or (the
    // instance for four CTAs per SM, within 128 registers) evaluated again in the sweep
    constexpr bool KEEP_E1 = ZOH && MINB < 4;
    constexpr int TT = Cfg::TT, N2 = 2 * N;
    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x, ng = tid % NG, dl = tid / NG;
    const int b = blockIdx.y, seg = p.seg0 + blockIdx.z;
    const int d0 = blockIdx.x * DT, d = d0 + dl, n0 = ng * Cfg::S;
    const bool dv = d < p.D;
    // slot rotation and the all-to-all partners among the four channel lanes of this group
    const int cl = (tid & 31) / NG, rot = A2A ? cl & 3 : 0, grp = dl >> 2;
    const int src1 = ng + NG * ((cl & ~3) | ((rot - 1) & 3));
    const int src2 = ng + NG * ((cl & ~3) | ((rot - 2) & 3));
    const int src3 = ng + NG * ((cl & ~3) | ((rot - 3) & 3));
    int sidx[4];  // state held by each slot
#pragma unroll
    for (int j = 0; j < 4; ++j) sidx[j] = n0 + ((j + rot) & 3);
    const int T = p.T;
    const int TTe = T < TT ? T : TT;
    const int c_begin = seg * p.seg_chunks;
    const int c_end = min(p.nC, c_begin + p.seg_chunks);

    float2 A[P2], A2[P2], v[P2], dA[P2];
    float2 Ar[P2];  // zero-order hold: 1 / A (the instance keeping E1; the other takes 1 / z per use)
    {
        const float* al = p.A_log + (size_t)(dv ? d : 0) * N;
#pragma unroll
        for (int i = 0; i < P2; ++i) {
            A[i] = dv ? make_float2(-expf(al[sidx[2 * i]]), -expf(al[sidx[2 * i + 1]]))
                      : make_float2(0.0f, 0.0f);
            A2[i] = __fmul2_rn(A[i], f2(kLog2e));
            if (ZOH)
                Ar[i] = dv ? make_float2(-expf(-al[sidx[2 * i]]), -expf(-al[sidx[2 * i + 1]]))
                           : make_float2(0.0f, 0.0f);
            v[i] = make_float2(0.0f, 0.0f);
            dA[i] = make_float2(0.0f, 0.0f);
        }
    }
    if (dv) {
        // the adjoint entering from the segment's end: handed over by the carry or by the later
        // block, or, for the last segment, the upstream gradient of the final state (or zero)
        const float* src = seg < p.nseg - 1 ? p.vin + (((size_t)b * (p.nseg - 1) + seg) * p.D + d) * N
                           : p.dhL          ? p.dhL + ((size_t)b * p.D + d) * N
                                            : nullptr;
        if (src) ld_slots(v, src, sidx);
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
    float* partb = p.dBC_part + ((size_t)blockIdx.x * p.B + b) * (size_t)p.part_rows * N2 -
                   (size_t)p.part_t0 * N2;  // indexed by absolute step t
    // scratch slot: the CTA's own index when the launch has no more CTAs than slots; else (POOL)
    // one claimed from the slot mask for the CTA's lifetime
    const int cta = (int)(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x);
    int slot = cta;
    if constexpr (POOL) {
        __shared__ int s_slot;
        if (tid == 0) s_slot = claim_slot(p.slot_mask, p.nslot, cta % p.nslot);
        __syncthreads();
        slot = s_slot;
        if (slot < 0) {  // no slot within the bound: this CTA's outputs stay unwritten, the call fails
            if (tid == 0) flag_status(p.status, kStatusTimeout);
            return;
        }
    }
    float* scr = p.bnd_scratch + (size_t)slot * real_bwd_scratch_floats(N, T);
    float* bnd = scr + (size_t)tid * 4;                        // window starts: [T/W][NT][4]
    float2* dsg = reinterpret_cast<float2*>(scr + (size_t)(T / W) * NT * 4);  // (delta, sigma) [T][DT]
    const int roff = rot * N + n0;  // this thread's slots within a staged row of ROT * N floats

    // fused dB/dC sums: the chunk whose sums are pending and this CTA's finished-chunk count
    static_assert(!FUSED || 2 * Sm::RED * 4 >= NT * 16, "the warps' part sums fit the window-sum buffer");
    int pend = -1, nfin = 0;
    unsigned* gcnt = FUSED ? p.grp_cnt + (size_t)seg * p.B + b : nullptr;
    auto sum_pending = [&]() {
        if constexpr (FUSED) {
            __shared__ int s_ok;
            if (tid == 0) {
                const unsigned target = (unsigned)nfin * (unsigned)p.ndt;
                unsigned it = 0;
                while (*reinterpret_cast<volatile unsigned*>(gcnt) < target && ++it < kSlotSpinLimit)
                    __nanosleep(128);
                s_ok = it < kSlotSpinLimit;
                __threadfence();  // the other CTAs' partial rows come first
                if (!s_ok) flag_status(p.status, kStatusTimeout);
            }
            __syncthreads();
            if (s_ok)
                fused_dbc_share<E, N>(p.dBC_part, p.part_rows, p.part_t0, p.B, p.L, p.T, p.ndt,
                                      static_cast<E*>(p.dB), static_cast<E*>(p.dC), b, pend,
                                      (int)blockIdx.x, tid, NT, reinterpret_cast<float4*>(smem + Sm::B_RED));
            pend = -1;
        }
    };

    for (int c = c_end - 1; c >= c_begin; --c) {
        const int tc = c * T;
        const int rows_c = min(T, p.L - tc);
        const int nsub = (rows_c + TTe - 1) / TTe;

        // ------------------------------------------------------------------ pass A
        {
            float2 h[P2];
            if (c > 0 && dv) {
                ld_slots(h, p.ckpt_in + (((size_t)b * p.nC + (c - 1)) * p.D + d) * N, sidx);
            } else if (p.h0 && dv) {
                ld_slots(h, p.h0 + ((size_t)b * p.D + d) * N, sidx);
            } else {
#pragma unroll
                for (int i = 0; i < P2; ++i) h[i] = make_float2(0.0f, 0.0f);
            }
            float2* sdd = reinterpret_cast<float2*>(smem + Sm::A_DD);
            float* sBr = reinterpret_cast<float*>(smem + Sm::A_BR);
            auto stage = [&](int k) { return reinterpret_cast<E*>(smem + k * Sm::A_STAGE); };
            auto issue = [&](int j, int k) {
                const int t0 = tc + j * TTe;
                E* sx = stage(k);
                cp_async_tile<E, DT>(sx, xb, t0, TTe, p.L, d0, p.D, tid, NT);
                cp_async_tile<E, DT>(sx + Sm::XE, drb, t0, TTe, p.L, d0, p.D, tid, NT);
                cp_async_flat<E>(sx + 2 * Sm::XE, Bb, (size_t)t0 * N, TTe * N, (size_t)p.L * N, tid, NT);
                cp_async_commit();
            };
            __syncthreads();  // previous users of the stage buffers are done
            issue(0, 0);
            for (int j = 0; j < nsub; ++j) {
                const int k = j & 1;
                cp_async_wait<0>();
                __syncthreads();  // sub-tile j is in; every thread is past sub-tile j-1
                if (j + 1 < nsub) issue(j + 1, k ^ 1);
                const int t0 = tc + j * TTe;
                const int rows = min(TTe, p.L - t0);
                const E* sx = stage(k);
                const E* sdr = sx + Sm::XE;
                const E* sB = sx + 2 * Sm::XE;
                // one exp per (t, d) gives delta and sigmoid; steps past the end get delta = 0
                for (int i = tid; i < TTe * DT; i += NT) {
                    const int r = i / DT;
                    float dlt = 0.0f, sig = 0.0f;
                    if (r < rows) {
                        const float z = Elem<E>::to_f(sdr[i]);
                        softplus_sigmoid(z, dlt, sig);
                    }
                    sdd[i] = make_float2(dlt, dlt * Elem<E>::to_f(sx[i]));
                    __stcg(&dsg[(size_t)(j * TTe) * DT + i], make_float2(dlt, sig));
                }
                rotate_rows<E, N, ROT>(sBr, sB, TTe, tid, NT);
                __syncthreads();
                for (int w = 0; w < TTe / W; ++w) {
                    __stcg(reinterpret_cast<float4*>(bnd + (size_t)((j * TTe) / W + w) * NT * 4),
                           make_float4(h[0].x, h[0].y, h[1].x, h[1].y));
#pragma unroll
                    for (int u = 0; u < W; ++u) {
                        const int r = w * W + u;
                        const float2 dd = sdd[r * DT + dl];
                        float2 bq[P2];
                        ld_pairs<4>(bq, sBr + r * ROT * N + roff);
#pragma unroll
                        for (int i = 0; i < P2; ++i) {
                            const float2 zl2 = __fmul2_rn(f2(dd.x), A2[i]);
                            const float2 a = ex2_pair(zl2);
                            float2 w = f2(dd.y);  // input weight times x: delta x, or phi x
                            if constexpr (ZOH)
                                w = __fmul2_rn(w, zoh_e1(__fmul2_rn(zl2, f2(kLn2)), a,
                                                         __fmul2_rn(f2(__fdividef(1.0f, dd.x)), Ar[i])));
                            h[i] = __ffma2_rn(a, h[i], __fmul2_rn(w, bq[i]));
                        }
                    }
                }
            }
        }

        if constexpr (FUSED) {
            if (pend >= 0) sum_pending();  // the previous chunk's sums, behind this pass A
        }

        // ------------------------------------------------------------------ pass B
        {
            float* sBr = reinterpret_cast<float*>(smem + Sm::B_BR);
            float* sCr = reinterpret_cast<float*>(smem + Sm::B_CR);
            float* sred = reinterpret_cast<float*>(smem + Sm::B_RED);
            auto stage = [&](int k) { return smem + k * Sm::B_STAGE; };
            auto issue = [&](int j, int k) {
                const int t0 = tc + j * TTe;
                unsigned char* st = stage(k);
                // (delta, sigma) of this chunk's rows, written by pass A (always in range)
                {
                    const float* src = reinterpret_cast<const float*>(dsg + (size_t)(j * TTe) * DT);
                    float* dst = reinterpret_cast<float*>(st);
                    for (int i = tid; i < TTe * DT * 2 / 4; i += NT)
                        cp_async16(dst + 4 * i, src + 4 * i, true);
                }
                E* sx = reinterpret_cast<E*>(st + Sm::XE * 8);
                cp_async_tile<E, DT>(sx, xb, t0, TTe, p.L, d0, p.D, tid, NT);
                cp_async_tile<E, DT>(sx + Sm::XE, dyb, t0, TTe, p.L, d0, p.D, tid, NT);
                cp_async_flat<E>(sx + 2 * Sm::XE, Bb, (size_t)t0 * N, TTe * N, (size_t)p.L * N, tid, NT);
                cp_async_flat<E>(sx + 2 * Sm::XE + Sm::BE, Cb, (size_t)t0 * N, TTe * N, (size_t)p.L * N, tid, NT);
                cp_async_commit();
            };
            __syncthreads();
            issue(nsub - 1, (nsub - 1) & 1);
            float2 hw[P2];  // state at the start of the next window to recompute
            ld_pairs_cg<4>(hw, bnd + (size_t)((nsub - 1) * TTe / W + TTe / W - 1) * NT * 4);
            for (int j = nsub - 1; j >= 0; --j) {
                const int k = j & 1;
                cp_async_wait<0>();
                __syncthreads();  // sub-tile j is in; every thread is past sub-tile j+1
                if (j > 0) issue(j - 1, k ^ 1);
                const int t0 = tc + j * TTe;
                const int rows = min(TTe, p.L - t0);
                const float2* sds = reinterpret_cast<const float2*>(stage(k));
                const E* sx = reinterpret_cast<const E*>(stage(k) + Sm::XE * 8);
                const E* sdy = sx + Sm::XE;
                const E* sB = sx + 2 * Sm::XE;
                const E* sC = sB + Sm::BE;
                rotate_rows<E, N, ROT>(sBr, sB, TTe, tid, NT);
                rotate_rows<E, N, ROT>(sCr, sC, TTe, tid, NT);
                __syncthreads();
                const int nw = TTe / W;  // 4 or 8 windows, even
                const int wbase = (j * TTe) / W;

                float2 aa[W][P2], pp[W][P2];  // (a_t, a_t h_{t-1}) of the current window
                // after a window's reverse sweep: outputs, then its dB/dC sums over the CTA
                auto finish_window = [&](int q, float (&sv)[SV * W], const float (&sbv)[W],
                                         const float (&scv)[W]) {
                    float* red = sred + (q & 1) * Sm::RED;
                    if constexpr (A2A) {
#pragma unroll
                        for (int u = 0; u < W; ++u) {
                            red[grp * RS + u * N2 + n0 + rot] = sbv[u];
                            red[grp * RS + u * N2 + N + n0 + rot] = scv[u];
                        }
                    } else {
                        // one lane per (dB or dC, state) writes the warp's sums of the window's
                        // steps: rows of 2N floats, a warp's lanes contiguous
                        const int lane = tid & 31, e = (lane >> 2) & 7;
                        if ((lane & 3 & ~(NG - 1)) == 0) {
                            float* wr = red + (tid >> 5) * W * N2 + (e >> 2) * N + ng * 4 + (e & 3);
#pragma unroll
                            for (int u = 0; u < W; ++u) wr[u * N2] = sbv[u];
                        }
                    }
                    reduce_scatter<SV * W, NG>(sv, ng);
#pragma unroll
                    for (int jj = 0; jj < W / NG; ++jj) {
                        const int uu = ng * (W / NG) + jj;
                        const int r = q * W + uu;
                        if (r < rows && dv) {
                            const float2 ds = sds[r * DT + dl];
                            const float xv = Elem<E>::to_f(sx[r * DT + dl]);
                            const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                            const float sgB = sv[SV * jj], sAq = sv[SV * jj + 1];
                            const float sgaB = ZOH ? sv[SV * jj + 2] : sgB;
                            const size_t o = (size_t)(t0 + r) * p.D + d;
                            dxb[o] = Elem<E>::from_f(fmaf(dsk, dyv, ds.x * sgB));
                            ddrb[o] = Elem<E>::from_f(fmaf(xv, sgaB, sAq) * ds.y);
                            dDacc = fmaf(dyv, xv, dDacc);
                        }
                    }
                    __syncthreads();  // every group's sums of the window are in `red`
                    {
                        // output (step u, dB or dC, state) = sum over the CTA's groups or warps
                        float s = 0.0f;
                        if constexpr (A2A) {
#pragma unroll
                            for (int g = 0; g < GRP; ++g) s += red[g * RS + tid];
                        } else {
                            const int u = tid / N2, e2 = tid % N2;
#pragma unroll
                            for (int w = 0; w < NT / 32; ++w) s += red[(w * W + u) * N2 + e2];
                        }
                        const int r = q * W + tid / N2;
                        if (r < rows) partb[(size_t)(t0 + r) * N2 + (tid % N2)] = s;
                    }
                };

                // windows in reverse: recompute (a_t, a_t h_{t-1}) forward from the window's start
                // state, keeping B_t, delta_t and delta_t x_t in registers for the reverse sweep
                for (int q = nw - 1; q >= 0; --q) {
                    float2 hc[P2] = {hw[0], hw[1]};
                    if (q >= 1) ld_pairs_cg<4>(hw, bnd + (size_t)(wbase + q - 1) * NT * 4);
                    float2 bqs[W][P2];
                    float2 e1s[KEEP_E1 ? W : 1][P2];  // zero-order hold: E1(delta A) per step
                    float dls[W], dxs[W], rds[KEEP_E1 ? W : 1];
#pragma unroll
                    for (int u = 0; u < W; ++u) {
                        const int r = q * W + u;
                        const float dlt = sds[r * DT + dl].x;
                        const float dxv = dlt * Elem<E>::to_f(sx[r * DT + dl]);
                        ld_pairs<4>(bqs[u], sBr + r * ROT * N + roff);
                        dls[u] = dlt;
                        dxs[u] = dxv;
                        if constexpr (KEEP_E1) rds[u] = __fdividef(1.0f, dlt);
#pragma unroll
                        for (int i = 0; i < P2; ++i) {
                            const float2 zl2 = __fmul2_rn(f2(dlt), A2[i]);
                            const float2 a = ex2_pair(zl2);
                            const float2 pr = __fmul2_rn(a, hc[i]);
                            aa[u][i] = a;
                            pp[u][i] = pr;
                            if constexpr (ZOH) {
                                const float2 z = __fmul2_rn(zl2, f2(kLn2));
                                const float2 e1 = zoh_e1(z, a, KEEP_E1 ? __fmul2_rn(f2(rds[u]), Ar[i]) : rcp_pair(z));
                                if constexpr (KEEP_E1) e1s[u][i] = e1;
                                hc[i] = __ffma2_rn(__fmul2_rn(f2(dxv), e1), bqs[u][i], pr);
                            } else {
                                hc[i] = __ffma2_rn(f2(dxv), bqs[u][i], pr);
                            }
                        }
                    }
                    float sv[SV * W];
                    float sbv[W], scv[W];  // this lane's state: dB, dC summed over its group, per step
#pragma unroll
                    for (int uu = W - 1; uu >= 0; --uu) {
                        const int r = q * W + uu;
                        const float dlt = dls[uu], dxv = dxs[uu];
                        const float dyv = Elem<E>::to_f(sdy[r * DT + dl]);
                        float2 cq[P2];
                        ld_pairs<4>(cq, sCr + r * ROT * N + roff);
                        float2 sg = make_float2(0.0f, 0.0f), sa = make_float2(0.0f, 0.0f);
                        float2 sga = make_float2(0.0f, 0.0f);
                        float2 rB[P2], rC[P2];
#pragma unroll
                        for (int i = 0; i < P2; ++i) {
                            const float2 g = __ffma2_rn(cq[i], f2(dyv), v[i]);      // adjoint g_t
                            const float2 qv = __fmul2_rn(g, pp[uu][i]);
                            dA[i] = __ffma2_rn(f2(dlt), qv, dA[i]);
                            sa = __ffma2_rn(A[i], qv, sa);
                            if constexpr (ZOH) {
                                // input weight phi = delta E1; d phi / ddelta = a;
                                // d phi / dA = delta^2 E2
                                const float2 z = __fmul2_rn(__fmul2_rn(f2(dlt), A2[i]), f2(kLn2));
                                const float2 rz = KEEP_E1 ? __fmul2_rn(f2(rds[uu]), Ar[i]) : rcp_pair(z);
                                float2 e1;
                                if constexpr (KEEP_E1)
                                    e1 = e1s[uu][i];
                                else
                                    e1 = zoh_e1(z, aa[uu][i], rz);  // as in the recompute
                                const float2 hj = __ffma2_rn(__fmul2_rn(f2(dxv), e1), bqs[uu][i],
                                                             pp[uu][i]);           // h_t
                                const float2 e2 = zoh_e2(z, aa[uu][i], e1, rz);
                                const float2 gb = __fmul2_rn(g, bqs[uu][i]);
                                dA[i] = __ffma2_rn(gb, __fmul2_rn(f2(dxv * dlt), e2), dA[i]);
                                sg = __ffma2_rn(gb, e1, sg);
                                rB[i] = __fmul2_rn(__fmul2_rn(g, e1), f2(dxv));
                                rC[i] = __fmul2_rn(f2(dyv), hj);
                                v[i] = __fmul2_rn(aa[uu][i], g);                    // a_t g_t
                                sga = __ffma2_rn(v[i], bqs[uu][i], sga);
                            } else {
                                const float2 hj = __ffma2_rn(f2(dxv), bqs[uu][i], pp[uu][i]);  // h_t
                                sg = __ffma2_rn(g, bqs[uu][i], sg);
                                rB[i] = __fmul2_rn(g, f2(dxv));
                                rC[i] = __fmul2_rn(f2(dyv), hj);
                                v[i] = __fmul2_rn(aa[uu][i], g);                    // a_t g_t
                            }
                        }
                        sv[SV * uu] = sg.x + sg.y;
                        sv[SV * uu + 1] = sa.x + sa.y;
                        if constexpr (ZOH) sv[SV * uu + 2] = sga.x + sga.y;
                        if constexpr (A2A) {
                            // all-to-all over the four channel lanes of the group: round k sends
                            // slot k, which the partner (rotation rot - k) holds for this lane's
                            // state
                            sbv[uu] = (rB[0].x + __shfl_sync(kFull, rB[0].y, src1)) +
                                      (__shfl_sync(kFull, rB[1].x, src2) + __shfl_sync(kFull, rB[1].y, src3));
                            scv[uu] = (rC[0].x + __shfl_sync(kFull, rC[0].y, src1)) +
                                      (__shfl_sync(kFull, rC[1].x, src2) + __shfl_sync(kFull, rC[1].y, src3));
                        } else {
                            // sum over the warp's channels (lane bits above the NG state lanes):
                            // the first three halvings scatter the 8 values (dB, dC of 4 states)
                            // so that lane element e = (lane >> 2) & 7 remains, further ones sum
                            float vv[8] = {rB[0].x, rB[0].y, rB[1].x, rB[1].y,
                                           rC[0].x, rC[0].y, rC[1].x, rC[1].y};
                            int c = 8;
#pragma unroll
                            for (int m = 16; m >= NG; m >>= 1) {
                                if (c > 1) {
                                    const bool up = (threadIdx.x & m) != 0;
                                    const int h = c / 2;
#pragma unroll
                                    for (int i2 = 0; i2 < 4; ++i2) {
                                        if (i2 < h) {
                                            const float send = up ? vv[i2] : vv[i2 + h];
                                            const float keep = up ? vv[i2 + h] : vv[i2];
                                            vv[i2] = keep + __shfl_xor_sync(kFull, send, m);
                                        }
                                    }
                                    c = h;
                                } else {
                                    vv[0] += __shfl_xor_sync(kFull, vv[0], m);
                                }
                            }
                            sbv[uu] = vv[0];
                            scv[uu] = 0.0f;
                        }
                    }
                    finish_window(q, sv, sbv, scv);
                }
                // state at the start of the last window of the previous sub-tile
                if (j > 0) ld_pairs_cg<4>(hw, bnd + (size_t)(wbase - 1) * NT * 4);
            }
        }
        if constexpr (FUSED) {
            __syncthreads();  // every partial row of chunk c is written
            if (tid == 0) {
                __threadfence();
                atomicAdd(gcnt, 1u);
            }
            pend = c;
            ++nfin;
        }
    }
    if constexpr (FUSED) {
        if (pend >= 0) sum_pending();
    }
    // each lane of a channel accumulated dD over its own subset of steps
#pragma unroll
    for (int m = 1; m < NG; m <<= 1) dDacc += __shfl_xor_sync(kFull, dDacc, m);
    if (dv) {
        const size_t o = (((size_t)b * p.nseg + seg) * p.D + d) * N;
        st_slots(p.dA_part + o, dA, sidx);
        if (ng == 0) p.dD_part[((size_t)b * p.nseg + seg) * p.D + d] = dDacc;
        // sequential blocks: the adjoint leaving this block's start enters the previous block
        if (p.seq_blocks && seg > 0)
            st_slots(p.vin + (((size_t)b * (p.nseg - 1) + (seg - 1)) * p.D + d) * N, v, sidx);
        // the first segment ends at t = -1: its adjoint a_0 g_0 is the gradient of h0
        if (p.dh0 && seg == 0) st_slots(p.dh0 + ((size_t)b * p.D + d) * N, v, sidx);
        if (!all_finite<4>(v)) flag_status(p.status, kStatusNonFinite);
    }
    if constexpr (POOL) {
        __syncthreads();  // every thread is done with the scratch slot
        if (tid == 0) {
            __threadfence();
            atomicAnd(p.slot_mask + slot / 32, ~(1u << (slot & 31)));
        }
    }
}

// dB, dC for the steps [part_t0, part_t0 + rows) of the current launch: fixed-order sums of the
// per-CTA partials over the channel tiles.
template <typename E, int N>
__global__ void real_reduce_dbc_kernel(RealArgs p, int rows) {
    constexpr int N2 = 2 * N;
    const int64_t total = (int64_t)p.B * rows * N2;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total) return;
    const int o = (int)(i % N2);
    const int64_t r = (i / N2) % rows;
    const int64_t b = i / ((int64_t)N2 * rows);
    const size_t stride = (size_t)p.B * p.part_rows * N2;
    const float* src = p.dBC_part + ((size_t)b * p.part_rows + r) * N2 + o;
    float s = 0.0f;
    for (int t = 0; t < p.ndt; ++t) s += src[(size_t)t * stride];
    const size_t bl = (size_t)b * p.L + p.part_t0 + r;
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

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Launch plan: segments [0, nseg) of seg_chunks chunks each.  Concurrent segments (seq_blocks
// == 0) get their entering adjoints from the summary + carry pass and run `group` segments per
// launch; sequential blocks (seq_blocks == 1) run one per launch from the end, each writing the
// adjoint entering the previous one.  Either way the dB/dC partial buffer holds the rows of one
// launch only, so its size does not grow with L.
template <typename E, int N, bool ZOH>
cudaError_t real_bwd_impl(const RealArgs& a0, int group, cudaStream_t st) {
    cudaError_t e;
    RealArgs a = a0;
    if (a.nseg > 1 && !a.seq_blocks) {
        a.seg0 = 1;
        const size_t sm = BwdSumSmem<E, N>::BYTES;
        if ((e = set_smem(real_bwd_summary_kernel<E, N, 4>, sm)) != cudaSuccess) return e;
        real_bwd_summary_kernel<E, N, 4><<<dim3(a.ndt, a.B, a.nseg - 1), dim3(RealCfg<N, 4>::NT), sm, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t n = (int64_t)a.B * a.D * N;
        real_carry_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.B, a.nseg, a.D * N,
                                                                            a.gsumP, a.vin, a.dhL);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // at most three CTAs per SM: the all-to-all instance; four: the reduce-scatter instance, whose
    // registers and shared memory fit four.  Instances: plain, claiming scratch slots (POOL, more
    // CTAs than slots), and with the fused dB/dC sums (FUSED, every CTA resident: cooperative)
    const size_t sm3 = BwdSmem<E, N, true>::BYTES, sm4 = BwdSmem<E, N, false>::BYTES;
    auto k3 = real_bwd_kernel<E, N, ZOH, 3, true, false, false>;
    auto k3p = real_bwd_kernel<E, N, ZOH, 3, true, true, false>;
    auto k3f = real_bwd_kernel<E, N, ZOH, 3, true, false, true>;
    if ((e = set_smem(k3, sm3)) != cudaSuccess || (e = set_smem(k3p, sm3)) != cudaSuccess ||
        (e = set_smem(k3f, sm3)) != cudaSuccess)
        return e;
    int dev = 0, sms = 0, coop = 0, res3 = 0, res4 = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&res3, k3f, BwdCfg<N>::NT, sm3)) != cudaSuccess)
        return e;
    if constexpr (N == 16) {
        auto k4 = real_bwd_kernel<E, N, ZOH, 4, false, false, false>;
        auto k4p = real_bwd_kernel<E, N, ZOH, 4, false, true, false>;
        auto k4f = real_bwd_kernel<E, N, ZOH, 4, false, false, true>;
        if ((e = set_smem(k4, sm4)) != cudaSuccess || (e = set_smem(k4p, sm4)) != cudaSuccess ||
            (e = set_smem(k4f, sm4)) != cudaSuccess)
            return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&res4, k4f, BwdCfg<N>::NT, sm4)) != cudaSuccess)
            return e;
    }
    const int per = a.seq_blocks ? 1 : group;
    for (int hi = a.nseg; hi > 0; hi -= per) {
        const int lo = hi - per > 0 ? hi - per : 0;
        a.seg0 = lo;
        a.part_t0 = lo * a.seg_chunks * a.T;
        const int t_hi = min(a.L, hi * a.seg_chunks * a.T);
        const int rows = t_hi - a.part_t0;
        const dim3 grid(a.ndt, a.B, hi - lo);
        const int64_t ctas = (int64_t)a.ndt * a.B * (hi - lo);
        const bool pool = ctas > a.nslot;  // more CTAs than scratch slots: claim them
        bool wide = false;                 // more CTAs than 3 per SM on 148 SMs
        if constexpr (N == 16) wide = ctas > 444;
        // asked for, and every CTA resident at once: the dB/dC sums run inside the scan kernel
        const bool fused = a.fused_sums && coop && !pool && ctas <= (int64_t)sms * (wide ? res4 : res3);
        const dim3 blk(BwdCfg<N>::NT);
        if (fused) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeCooperative;
            attr[0].val.cooperative = 1;
            cfg.gridDim = grid;
            cfg.blockDim = blk;
            cfg.stream = st;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (wide) {
                if constexpr (N == 16) {
                    cfg.dynamicSmemBytes = sm4;
                    e = cudaLaunchKernelEx(&cfg, real_bwd_kernel<E, N, ZOH, 4, false, false, true>, a);
                }
            } else {
                cfg.dynamicSmemBytes = sm3;
                e = cudaLaunchKernelEx(&cfg, k3f, a);
            }
            if (e != cudaSuccess) return e;
            continue;  // dB and dC are written: no reduction launch
        }
        if (wide) {
            if constexpr (N == 16) {
                if (pool)
                    real_bwd_kernel<E, N, ZOH, 4, false, true, false><<<grid, blk, sm4, st>>>(a);
                else
                    real_bwd_kernel<E, N, ZOH, 4, false, false, false><<<grid, blk, sm4, st>>>(a);
            }
        } else if (pool) {
            k3p<<<grid, blk, sm3, st>>>(a);
        } else {
            k3<<<grid, blk, sm3, st>>>(a);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t nbc = (int64_t)a.B * rows * 2 * N;
        if (nbc > 0) {
            real_reduce_dbc_kernel<E, N><<<(unsigned)((nbc + 255) / 256), 256, 0, st>>>(a, rows);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    const int64_t np = (int64_t)a.D * N;
    real_reduce_params_kernel<<<(unsigned)((np + 255) / 256), 256, 0, st>>>(a, N);
    return cudaGetLastError();
}

template <typename E, bool ZOH>
cudaError_t bwd_dispatch_n(const RealArgs& a, int N, int group, cudaStream_t st) {
    if (N == 4) return real_bwd_impl<E, 4, ZOH>(a, group, st);
    if (N == 8) return real_bwd_impl<E, 8, ZOH>(a, group, st);
    return real_bwd_impl<E, 16, ZOH>(a, group, st);
}

template <typename E>
cudaError_t bwd_dispatch(const RealArgs& a, int N, int group, cudaStream_t st) {
    return a.zoh ? bwd_dispatch_n<E, true>(a, N, group, st) : bwd_dispatch_n<E, false>(a, N, group, st);
}

}  // namespace
}  // namespace real

cudaError_t launch_real_bwd(const RealArgs& a, int io_bf16, int N, int group, cudaStream_t st) {
    return io_bf16 ? real::bwd_dispatch<__nv_bfloat16>(a, N, group, st)
                   : real::bwd_dispatch<float>(a, N, group, st);
}

}  // namespace ssm
