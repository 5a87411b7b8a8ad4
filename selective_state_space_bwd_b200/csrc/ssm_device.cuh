// Device-side helpers shared by the scan kernels: element conversion, 16-byte tile movers,
// the discretisation functions and the status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Status codes written into the workspace status word (mirror of ssm_status in ssm_scan.h).
constexpr unsigned kStatusTimeout = 6u;
constexpr unsigned kStatusNonFinite = 7u;

__device__ __forceinline__ void flag_status(unsigned* status, unsigned code) {
    atomicCAS(status, 0u, code);  // first condition wins
}

// 2^x on the MUFU unit (PTX ex2.approx.ftz.f32): relative error ~2^-22, flushes denormals.
__device__ __forceinline__ float ex2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(z) = max(z, 0) + log1p(exp(-|z|)), the step-size map of the selective SSM.
__device__ __forceinline__ float softplus_acc(float z) {
    return fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z)));
}

// softplus(z) = max(z, 0) + log1p(e), e = exp(-|z|) in [0, 1], using the identity
// log1p(e) = 2 atanh(s) with s = e / (2 + e) in [0, 1/3] and a polynomial in w = s^2 for
// 2 atanh(s) / s, fitted here (iteratively reweighted least squares towards minimax, max relative
// error 4.5e-9 on [0, 1/9]).  With the MUFU exp2 the result is within ~6e-7 relative of softplus.
__device__ __forceinline__ float softplus_fast(float z) {
    const float e = ex2_mufu(-fabsf(z) * kLog2e);
    const float s = __fdividef(e, 2.0f + e);
    const float w = s * s;
    float q = fmaf(w, 0.28011780977249146f, 0.2800184488296509f);
    q = fmaf(w, q, 0.4002152383327484f);
    q = fmaf(w, q, 0.666664183139801f);
    q = fmaf(w, q, 2.0f);
    return fmaf(s, q, fmaxf(z, 0.0f));
}

// softplus(z) and sigmoid(z) = d softplus / dz from one shared exp(-|z|).
__device__ __forceinline__ void softplus_sigmoid(float z, float& sp, float& sg) {
    const float e = ex2_mufu(-fabsf(z) * kLog2e);
    const float s = __fdividef(e, 2.0f + e);
    const float w = s * s;
    float q = fmaf(w, 0.28011780977249146f, 0.2800184488296509f);
    q = fmaf(w, q, 0.4002152383327484f);
    q = fmaf(w, q, 0.666664183139801f);
    q = fmaf(w, q, 2.0f);
    sp = fmaf(s, q, fmaxf(z, 0.0f));
    const float r = __fdividef(1.0f, 1.0f + e);
    sg = z >= 0.0f ? r : e * r;
}

// sigmoid(z) = 1 / (1 + exp(-z)) from e = exp(-|z|); within ~5e-7 relative.
__device__ __forceinline__ float sigmoid_fast(float z) {
    const float e = ex2_mufu(-fabsf(z) * kLog2e);
    const float r = __fdividef(1.0f, 1.0f + e);
    return z >= 0.0f ? r : e * r;
}

// sigmoid(z) = d softplus / dz, evaluated without overflow for either sign of z.
__device__ __forceinline__ float sigmoid_acc(float z) {
    const float e = expf(-fabsf(z));
    const float s = 1.0f / (1.0f + e);
    return z >= 0.0f ? s : e * s;
}

// ---------------------------------------------------------------- element conversion
template <typename E> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------- 16-byte tile movers
// Copy rows [t0, t0 + rows) x columns [c0, c0 + COLS) of a row-major [*, ncol] array into
// dst[rows][COLS]; rows at or past `nrow` and columns at or past `ncol` read as zero.  ncol must be
// a multiple of 16 / sizeof(E) (the host validates this), so every 16-byte vector is wholly in or
// wholly out of range.
template <typename E, int COLS>
__device__ __forceinline__ void load_tile(E* __restrict__ dst, const E* __restrict__ src, int t0,
                                          int rows, int nrow, int c0, int ncol, int tid,
                                          int nthreads) {
    constexpr int VEC = 16 / sizeof(E);
    constexpr int VPR = COLS / VEC;
    static_assert(COLS % VEC == 0, "tile width must be whole 16-byte vectors");
    for (int i = tid; i < rows * VPR; i += nthreads) {
        const int r = i / VPR, v = i - r * VPR;
        const int t = t0 + r, c = c0 + v * VEC;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (t < nrow && c < ncol)
            val = __ldg(reinterpret_cast<const uint4*>(src + (size_t)t * ncol + c));
        *reinterpret_cast<uint4*>(dst + r * COLS + v * VEC) = val;
    }
}

// Inverse of load_tile: write src[rows][COLS] back, skipping out-of-range rows / columns.
template <typename E, int COLS>
__device__ __forceinline__ void store_tile(E* __restrict__ dst, const E* __restrict__ src, int t0,
                                           int rows, int nrow, int c0, int ncol, int tid,
                                           int nthreads) {
    constexpr int VEC = 16 / sizeof(E);
    constexpr int VPR = COLS / VEC;
    for (int i = tid; i < rows * VPR; i += nthreads) {
        const int r = i / VPR, v = i - r * VPR;
        const int t = t0 + r, c = c0 + v * VEC;
        if (t < nrow && c < ncol)
            *reinterpret_cast<uint4*>(dst + (size_t)t * ncol + c) =
                *reinterpret_cast<const uint4*>(src + r * COLS + v * VEC);
    }
}

// Load `rows` consecutive rows of N elements (a [*, N] array, rows starting at t0) into a float
// tile dst[rows][N], zero past `nrow`.
template <typename E, int N>
__device__ __forceinline__ void load_rows_f32(float* __restrict__ dst, const E* __restrict__ src,
                                              int t0, int rows, int nrow, int tid, int nthreads) {
    for (int i = tid; i < rows * N; i += nthreads) {
        const int r = i / N;
        const int t = t0 + r;
        dst[i] = t < nrow ? Elem<E>::to_f(src[(size_t)t0 * N + i]) : 0.0f;
    }
}

}  // namespace ssm
