// Device helpers shared by the real-mode forward and backward kernels.
#pragma once

#include "ssm_device.cuh"
#include "ssm_internal.h"

namespace ssm {
namespace real {

constexpr unsigned kFull = 0xffffffffu;

template <int N, int S_>
struct RealCfg {
    static constexpr int S = S_;            // states per thread
    static constexpr int P2 = S / 2;        // state pairs per thread
    static constexpr int NG = N / S;        // lanes per channel
    static constexpr int DT = kRealDT;      // channels per CTA
    static constexpr int NT = DT * NG;      // threads per CTA
    static constexpr int TS = S == 4 ? 8 : 4;  // backward window: steps of (a, a h_prev) in registers
    static constexpr int U = 4;             // steps per unrolled group (= dB/dC flush period)
    static constexpr int Q = NT / (2 * N);  // channel parts in the dB/dC column sums
    static_assert(S == 4 || S == 8, "states per thread");
    static_assert(N % S == 0 && NG >= 1 && NG <= 4, "dstate must be 4, 8 or 16");
    static_assert(Q >= 1 && (DT % Q) == 0, "column-sum split");
};

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// exp2 of both halves on the MUFU unit
__device__ __forceinline__ float2 ex2_pair(float2 e) { return make_float2(ex2_mufu(e.x), ex2_mufu(e.y)); }

// S consecutive floats from shared / global memory as S/2 pairs (16-byte vector accesses; one
// 8-byte access for S = 2)
template <int S>
__device__ __forceinline__ void ld_pairs(float2 (&o)[S / 2], const float* p) {
    if constexpr (S == 2) {
        o[0] = *reinterpret_cast<const float2*>(p);
    } else {
#pragma unroll
        for (int i = 0; i < S / 4; ++i) {
            const float4 v = reinterpret_cast<const float4*>(p)[i];
            o[2 * i] = make_float2(v.x, v.y);
            o[2 * i + 1] = make_float2(v.z, v.w);
        }
    }
}
template <int S>
__device__ __forceinline__ void st_pairs(float* p, const float2 (&o)[S / 2]) {
    if constexpr (S == 2) {
        *reinterpret_cast<float2*>(p) = o[0];
    } else {
#pragma unroll
        for (int i = 0; i < S / 4; ++i)
            reinterpret_cast<float4*>(p)[i] =
                make_float4(o[2 * i].x, o[2 * i].y, o[2 * i + 1].x, o[2 * i + 1].y);
    }
}
template <int S>
__device__ __forceinline__ void st_pairs_cg(float* p, const float2 (&o)[S / 2]) {
#pragma unroll
    for (int i = 0; i < S / 4; ++i)
        __stcg(reinterpret_cast<float4*>(p) + i,
               make_float4(o[2 * i].x, o[2 * i].y, o[2 * i + 1].x, o[2 * i + 1].y));
}
template <int S>
__device__ __forceinline__ void ld_pairs_cg(float2 (&o)[S / 2], const float* p) {
#pragma unroll
    for (int i = 0; i < S / 4; ++i) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p) + i);
        o[2 * i] = make_float2(v.x, v.y);
        o[2 * i + 1] = make_float2(v.z, v.w);
    }
}

template <int S>
__device__ __forceinline__ bool all_finite(const float2 (&v)[S / 2]) {
    bool ok = true;
#pragma unroll
    for (int i = 0; i < S / 2; ++i) ok = ok && isfinite(v[i].x) && isfinite(v[i].y);
    return ok;
}

// ---------------------------------------------------------------- zero-order hold
// For a pair of exponents z = delta * A <= 0 (natural units), with a = exp(z) and rz = 1 / z:
//   E1(z) = expm1(z) / z           the input weight is phi = (exp(delta A) - 1) / A = delta E1(z)
//   E2(z) = (exp(z) - E1(z)) / z   d phi / dA = (delta a - phi) / A = delta^2 E2(z)
// Below |z| = 1/4 both come from their Taylor series about 0 (E1 = sum_k z^k / (k+1)!,
// E2 = sum_k z^(k-1) k / (k+1)!), six terms each: the first omitted terms, z^6 / 5040 and
// z^6 / 5760, are under 1.1e-7 of E1 and E2 there.  From |z| = 1/4 on they come from the
// quotients: a's relative error (about 2^-22 from the exp2 unit) then costs E1 at most
// 2.4e-7 / (0.25 * 0.88) = 1.1e-6 relative and E2, through a - E1 >= 0.1, about 1.2e-5.  delta = 0
// (padding) gives rz = inf and z = 0, which selects the series.
constexpr float kZohSeries = -0.25f;

// 1 / z of a pair (fast reciprocal; only the quotient branch, |z| >= 1/4, uses it)
__device__ __forceinline__ float2 rcp_pair(float2 z) {
    return make_float2(__fdividef(1.0f, z.x), __fdividef(1.0f, z.y));
}

__device__ __forceinline__ float2 zoh_e1(float2 z, float2 a, float2 rz) {
    float2 p = f2(1.0f / 720.0f);
    p = __ffma2_rn(p, z, f2(1.0f / 120.0f));
    p = __ffma2_rn(p, z, f2(1.0f / 24.0f));
    p = __ffma2_rn(p, z, f2(1.0f / 6.0f));
    p = __ffma2_rn(p, z, f2(0.5f));
    p = __ffma2_rn(p, z, f2(1.0f));
    const float2 q = __fmul2_rn(__fadd2_rn(a, f2(-1.0f)), rz);
    return make_float2(z.x > kZohSeries ? p.x : q.x, z.y > kZohSeries ? p.y : q.y);
}

__device__ __forceinline__ float2 zoh_e2(float2 z, float2 a, float2 e1, float2 rz) {
    float2 p = f2(1.0f / 840.0f);
    p = __ffma2_rn(p, z, f2(1.0f / 144.0f));
    p = __ffma2_rn(p, z, f2(1.0f / 30.0f));
    p = __ffma2_rn(p, z, f2(1.0f / 8.0f));
    p = __ffma2_rn(p, z, f2(1.0f / 3.0f));
    p = __ffma2_rn(p, z, f2(0.5f));
    const float2 q = __fmul2_rn(__ffma2_rn(e1, f2(-1.0f), a), rz);
    return make_float2(z.x > kZohSeries ? p.x : q.x, z.y > kZohSeries ? p.y : q.y);
}

// Reduce-scatter of V per-lane values over the NG adjacent lanes of a channel: on return lane
// `ng` holds, in v[0 .. V/NG), the channel totals of values [ng*V/NG, (ng+1)*V/NG).
template <int V, int NG>
__device__ __forceinline__ void reduce_scatter(float (&v)[V], int ng) {
    int c = V;
#pragma unroll
    for (int m = NG / 2; m >= 1; m >>= 1) {
        const bool up = (ng & m) != 0;
        const int h = c / 2;
#pragma unroll
        for (int i = 0; i < V / 2; ++i) {
            if (i < h) {
                const float send = up ? v[i] : v[i + h];
                const float keep = up ? v[i + h] : v[i];
                v[i] = keep + __shfl_xor_sync(kFull, send, m);
            }
        }
        c = h;
    }
}


// ---------------------------------------------------------------- asynchronous copies (LDGSTS)
// 16 bytes global -> shared; with valid == false nothing is read and the destination is zeroed.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, bool valid) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int PENDING>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(PENDING));
}

// Asynchronously copy rows [t0, t0 + rows) x columns [c0, c0 + COLS) of a row-major [*, ncol]
// array into dst[rows][COLS]; out-of-range rows / columns are zero-filled.  ncol is a multiple of
// 16 / sizeof(E), so every 16-byte vector is wholly in or out of range.
template <typename E, int COLS>
__device__ __forceinline__ void cp_async_tile(E* __restrict__ dst, const E* __restrict__ src, int t0,
                                              int rows, int nrow, int c0, int ncol, int tid,
                                              int nthreads) {
    constexpr int VEC = 16 / sizeof(E);
    constexpr int VPR = COLS / VEC;
    static_assert(COLS % VEC == 0, "tile width must be whole 16-byte vectors");
    for (int i = tid; i < rows * VPR; i += nthreads) {
        const int r = i / VPR, v = i - r * VPR;
        const int t = t0 + r, c = c0 + v * VEC;
        const bool ok = t < nrow && c < ncol;
        cp_async16(dst + r * COLS + v * VEC, ok ? src + (size_t)t * ncol + c : src, ok);
    }
}

// 1-D asynchronous copy of elements [e0, e0 + ne) of a contiguous array of `etotal` elements,
// zero-filling past the end.  ne * sizeof(E) is a multiple of 16.  The pieces are 16 bytes when
// the source start is 16-byte aligned, else 8 or 4 bytes (a [B, L, N] bf16 array with N = 4 and
// odd L starts odd batch rows on an 8-byte boundary).
template <int G, typename E>
__device__ __forceinline__ void cp_async_pieces(E* __restrict__ dst, const E* __restrict__ src,
                                                size_t e0, int ne, size_t etotal, int tid,
                                                int nthreads) {
    constexpr int VEC = G / sizeof(E);
    for (int i = tid; i < ne / VEC; i += nthreads) {
        const size_t e = e0 + (size_t)i * VEC;
        const size_t left = e < etotal ? etotal - e : 0;
        const int bytes = left >= (size_t)VEC ? G : (int)(left * sizeof(E));
        const unsigned s = (unsigned)__cvta_generic_to_shared(dst + i * VEC);
        const E* g = bytes > 0 ? src + e : src;
        if (G == 16)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(g), "r"(bytes));
        else if (G == 8)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(s), "l"(g), "r"(bytes));
        else
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(g), "r"(bytes));
    }
}
template <typename E>
__device__ __forceinline__ void cp_async_flat(E* __restrict__ dst, const E* __restrict__ src,
                                              size_t e0, int ne, size_t etotal, int tid,
                                              int nthreads) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(src + e0);
    if ((a & 15) == 0)
        cp_async_pieces<16>(dst, src, e0, ne, etotal, tid, nthreads);
    else if ((a & 7) == 0)
        cp_async_pieces<8>(dst, src, e0, ne, etotal, tid, nthreads);
    else
        cp_async_pieces<4>(dst, src, e0, ne, etotal, tid, nthreads);
}

}  // namespace real
}  // namespace ssm
