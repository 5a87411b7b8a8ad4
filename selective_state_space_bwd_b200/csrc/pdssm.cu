// Flash PD-SSM scan ("Flash PD-SSM: Memory-Optimized Structured Sparse State-Space Models",
// technical summary, sections 1-2: hard selection of one of K precomputed sparse dictionary
// matrices per step by argmax of input-generated scores; straight-through gradients with a
// tempered softmax in the backward pass).  Per batch b and head e, a real state h in R^N:
//   k_t = argmax_k scores_t[k] (ties: lowest k),   h_t = P_{k_t} D_t h_{t-1} + bt_t,
// P_k a one-hot column selector (column j has its 1 in row dict[k][j]), D_t = diag(d_t).
// Backward (L = sum_t <g_t, h_t>): mu_t = g_t + A_{t+1}^T mu_{t+1}, (A^T mu)_j = d_j mu[dict[k][j]];
//   dbt = mu, dd_t[j] = mu_t[dict[k_t][j]] h_{t-1}[j], dh0 = A_0^T mu_0,
//   dscores_t[k] = p_k (c_k - sum p c) / tau,  c_k = <mu_t, P_k D_t h_{t-1}>,  p = softmax(scores_t / tau).
//
// Layout [B, L, H, N] (state fastest): a CTA takes kPdThreads / N consecutive heads of one batch
// row, lane j of each N-lane group owns state j, so one step of the CTA reads and writes one
// contiguous 512-byte row.  The scatter of P (several columns may land on one row) goes through
// shared memory with per-row source lists built from the dictionary (ascending source order, so
// sums are deterministic); the backward's gather needs no lists.  Tiles of steps stream through
// two-stage cp.async rings.  The selection (argmax) and the score gradient are separate kernels,
// parallel over (b, t, e).
#include "real_common.cuh"

namespace ssm {
namespace {

using real::cp_async_commit;
using real::cp_async_flat;
using real::cp_async_wait;

constexpr int NT = kPdThreads;
constexpr int KMAX = 32;  // dictionary size limit (validated on the host)

// sel[b,t,e] = argmax_k scores[b,t,e,k], lowest index on ties.
__global__ void pdssm_select_kernel(PdArgs p) {
    const int64_t n = (int64_t)p.B * p.L * p.H;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float* sc = p.scores + i * p.K;
    int kb = 0;
    float best = sc[0];
    for (int k = 1; k < p.K; ++k) {
        const float v = sc[k];
        if (v > best) {
            best = v;
            kb = k;
        }
    }
    p.sel[i] = kb;
}

// Copy the rows t0 .. t0+TT-1 of one CTA (NT consecutive floats per row, row stride H*N floats)
// of a [B, L, H, N] array into dst[TT][NT], 16 bytes per piece; pieces past the array end read as
// zero (rows past L of a batch row are never used).
template <int TT>
__device__ __forceinline__ void tile_rows(float* dst, const float* src, size_t first, size_t stride,
                                          size_t total, int tid) {
    constexpr int PR = NT / 4;  // pieces per row
#pragma unroll
    for (int q = tid; q < TT * PR; q += NT) {
        const int r = q / PR, c = q - r * PR;
        const size_t e = first + (size_t)r * stride + 4 * c;
        const bool ok = e + 4 <= total;
        real::cp_async16(dst + r * NT + 4 * c, ok ? src + e : src, ok);
    }
}

// The same for the int32 selection, one (b, t, e) entry per 4-byte piece.
template <int TT, int SEQ>
__device__ __forceinline__ void tile_sel(int* dst, const int32_t* src, size_t first, size_t stride,
                                         size_t total, int tid) {
    for (int q = tid; q < TT * SEQ; q += NT) {
        const int r = q / SEQ, c = q - r * SEQ;
        const size_t e = first + (size_t)r * stride + c;
        const unsigned sa = (unsigned)__cvta_generic_to_shared(dst + q);
        const int n = e < total ? 4 : 0;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(sa),
                     "l"(n ? src + e : src), "r"(n));
    }
}

// Dictionary entry, clamped into [0, N); an entry out of range sets SSM_ERR_INVALID_ARG (1) in
// the status word (the host cannot see device memory before launching).
template <int N>
__device__ __forceinline__ int dict_row(const int32_t* dict, int i, unsigned* status) {
    const int v = dict[i];
    if (v < 0 || v >= N) {
        flag_status(status, 1u);
        return v < 0 ? 0 : N - 1;
    }
    return v;
}

// In-lists of the dictionary: for matrix k and row i, the columns j with dict[k][j] == i, in
// ascending j, at src[k*N + start[k*(N+1) + i] ...].
template <int N>
__device__ __forceinline__ void build_lists(const int32_t* dict, int K, unsigned char* start,
                                            unsigned char* src, int tid, unsigned* status) {
    for (int k = tid; k < K; k += NT) {
        int cnt[N];
#pragma unroll
        for (int i = 0; i < N; ++i) cnt[i] = 0;
        for (int j = 0; j < N; ++j) ++cnt[dict_row<N>(dict, k * N + j, status)];
        int acc = 0;
#pragma unroll
        for (int i = 0; i < N; ++i) {
            start[k * (N + 1) + i] = (unsigned char)acc;
            acc += cnt[i];
            cnt[i] = start[k * (N + 1) + i];
        }
        start[k * (N + 1) + N] = (unsigned char)acc;
        for (int j = 0; j < N; ++j) src[k * N + cnt[dict_row<N>(dict, k * N + j, status)]++] = (unsigned char)j;
    }
}

// Padded source table: every row gets the same number D of entries (the largest in-degree of the
// dictionary), the missing ones pointing at slot N of its group, which holds zero.  With it every
// lane of the scatter loops D times, so the lanes of a warp do not diverge.  Returns D, or 0 when
// the table would not fit in PAD_BYTES (then the lists are used as they are).
constexpr int PAD_BYTES = 4096;

template <int N>
__device__ __forceinline__ int build_pad(const unsigned char* start, const unsigned char* src, int K,
                                         unsigned char* pad, int* s_deg, int tid) {
    if (tid == 0) *s_deg = 0;
    __syncthreads();
    for (int i = tid; i < K * N; i += NT) {
        const int k = i / N, r = i - k * N;
        atomicMax(s_deg, start[k * (N + 1) + r + 1] - start[k * (N + 1) + r]);
    }
    __syncthreads();
    const int D = *s_deg;
    if (D == 0 || K * N * D > PAD_BYTES) return 0;
    for (int i = tid; i < K * N; i += NT) {
        const int k = i / N, r = i - k * N;
        const int a = start[k * (N + 1) + r], c = start[k * (N + 1) + r + 1] - a;
        for (int m = 0; m < D; ++m) pad[i * D + m] = m < c ? src[k * N + a + m] : (unsigned char)N;
    }
    __syncthreads();
    return D;
}

template <int N>
__global__ void __launch_bounds__(NT) pdssm_fwd_kernel(PdArgs p) {
    constexpr int SEQ = NT / N, TT = 16;
    __shared__ __align__(16) float sd[2][TT * NT];
    __shared__ __align__(16) float sb[2][TT * NT];
    __shared__ __align__(16) int ssel[2][TT * SEQ];
    __shared__ float sv[SEQ * (N + 1)];  // per group: N values and a zero slot
    __shared__ unsigned char s_start[KMAX * (N + 1)];
    __shared__ unsigned char s_src[KMAX * N];
    __shared__ unsigned char s_pad[PAD_BYTES];
    __shared__ int s_deg;
    const int tid = threadIdx.x, j = tid % N, sq = tid / N;
    const int b = blockIdx.y, e0 = blockIdx.x * SEQ, e = e0 + sq;
    const bool ev = e < p.H;
    const size_t total = (size_t)p.B * p.L * p.H;  // (b, t, e) rows
    build_lists<N>(p.dict, p.K, s_start, s_src, tid, p.status);
    if (j == 0) sv[sq * (N + 1) + N] = 0.0f;
    __syncthreads();
    const int D = build_pad<N>(s_start, s_src, p.K, s_pad, &s_deg, tid);
    float* svg = sv + sq * (N + 1);
    const int seg = blockIdx.z;
    const int t_begin = seg * p.seg_len, t_end = min(p.L, t_begin + p.seg_len);
    float h = 0.0f;
    if (ev) {
        if (p.nseg > 1)
            h = p.hin[(((size_t)b * p.H + e) * p.nseg + seg) * N + j];
        else if (p.h0)
            h = p.h0[((size_t)b * p.H + e) * N + j];
    }
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    auto row0 = [&](int t) { return ((size_t)b * p.L + t) * p.H + e0; };  // first (b,t,e) row
    const size_t rstride = (size_t)p.H * N;
    auto issue = [&](int jt, int st) {
        const size_t o = row0(t_begin + jt * TT);
        tile_rows<TT>(sd[st], p.d, o * N, rstride, total * N, tid);
        tile_rows<TT>(sb[st], p.bt, o * N, rstride, total * N, tid);
        tile_sel<TT, SEQ>(ssel[st], p.sel, o, p.H, total, tid);
        cp_async_commit();
    };
    __syncthreads();  // dictionary lists
    if (ntiles > 0) issue(0, 0);
    for (int jt = 0; jt < ntiles; ++jt) {
        const int st = jt & 1;
        if (jt + 1 < ntiles) {
            issue(jt + 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int t0 = t_begin + jt * TT, rows = min(TT, t_end - t0);
        float* hout = p.h + (row0(t0) + sq) * N + j;
        const size_t hstep = (size_t)p.H * N;
        for (int r = 0; r < rows; ++r) {
            const int k = min(max(ssel[st][r * SEQ + sq], 0), p.K - 1);
            svg[j] = sd[st][r * NT + tid] * h;
            __syncwarp();
            float acc = sb[st][r * NT + tid];
            if (D > 0) {  // uniform trip count: no divergence
                const unsigned char* row = s_pad + (k * N + j) * D;
                for (int m = 0; m < D; ++m) acc += svg[row[m]];
            } else {
                const int q1 = s_start[k * (N + 1) + j + 1];
                for (int q = s_start[k * (N + 1) + j]; q < q1; ++q) acc += svg[s_src[k * N + q]];
            }
            h = acc;
            if (ev) *hout = h;
            hout += hstep;
            __syncwarp();
        }
        __syncthreads();  // stage st is free again
    }
    if (ev && !isfinite(h)) flag_status(p.status, kStatusNonFinite);
}

template <int N>
__global__ void __launch_bounds__(NT) pdssm_bwd_kernel(PdArgs p) {
    constexpr int SEQ = NT / N, TT = 8;
    __shared__ __align__(16) float sg[2][TT * NT];
    __shared__ __align__(16) float sd[2][TT * NT];
    __shared__ __align__(16) float shp[2][TT * NT];  // h_{t-1} of the tile's steps
    __shared__ __align__(16) int ssel[2][TT * SEQ];
    __shared__ float sv[NT];
    __shared__ unsigned char s_dict[KMAX * N];
    const int tid = threadIdx.x, j = tid % N, sq = tid / N;
    const int b = blockIdx.y, e0 = blockIdx.x * SEQ, e = e0 + sq;
    const bool ev = e < p.H;
    const size_t total = (size_t)p.B * p.L * p.H;
    for (int i = tid; i < p.K * N; i += NT) s_dict[i] = (unsigned char)dict_row<N>(p.dict, i, p.status);
    const int seg = blockIdx.z;
    const int t_begin = seg * p.seg_len, t_end = min(p.L, t_begin + p.seg_len);
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    auto row0 = [&](int t) { return ((size_t)b * p.L + t) * p.H + e0; };
    const size_t rstride = (size_t)p.H * N;
    auto issue = [&](int jt, int st) {
        const int t0 = t_begin + jt * TT;
        const size_t o = row0(t0);
        tile_rows<TT>(sg[st], p.g, o * N, rstride, total * N, tid);
        tile_rows<TT>(sd[st], p.d, o * N, rstride, total * N, tid);
        tile_sel<TT, SEQ>(ssel[st], p.sel, o, p.H, total, tid);
        if (t0 > 0) {
            tile_rows<TT>(shp[st], p.h, (o - p.H) * N, rstride, total * N, tid);
        } else {  // row 0 is h_{-1} = h0 (or zero), rows 1.. the trajectory
            tile_rows<TT - 1>(shp[st] + NT, p.h, o * N, rstride, total * N, tid);
            if (p.h0) {
                const size_t bh = (size_t)p.B * p.H * N;
                cp_async_flat<float>(shp[st], p.h0, ((size_t)b * p.H + e0) * N, NT, bh, tid, NT);
            } else {
                shp[st][tid] = 0.0f;
            }
        }
        cp_async_commit();
    };
    __syncthreads();  // dictionary
    float w = 0.0f;   // A_{t+1}^T mu_{t+1}: from the carry (or later segment), zero at the end
    if (ev && seg < p.nseg - 1) w = p.win[(((size_t)b * p.H + e) * p.nseg + seg) * N + j];
    if (ntiles > 0) issue(ntiles - 1, (ntiles - 1) & 1);
    for (int jt = ntiles - 1; jt >= 0; --jt) {
        const int st = jt & 1;
        if (jt > 0) {
            issue(jt - 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int t0 = t_begin + jt * TT, rows = min(TT, t_end - t0);
        const size_t base = (row0(t0) + sq) * N + j;
        for (int r = rows - 1; r >= 0; --r) {
            const int k = min(max(ssel[st][r * SEQ + sq], 0), p.K - 1);
            const float mu = sg[st][r * NT + tid] + w;
            sv[tid] = mu;
            __syncwarp();
            const float m = sv[sq * N + s_dict[k * N + j]];
            if (ev) {
                const size_t o = base + (size_t)r * p.H * N;
                p.dbt[o] = mu;
                p.dd[o] = m * shp[st][r * NT + tid];
            }
            w = sd[st][r * NT + tid] * m;
            __syncwarp();
        }
        __syncthreads();  // stage st is free again
    }
    if (ev) {
        if (p.dh0 && seg == 0) p.dh0[((size_t)b * p.H + e) * N + j] = w;
        if (!isfinite(w)) flag_status(p.status, kStatusNonFinite);
    }
}

// Phase A of the forward (segments 0..nseg-2): the scan of the segment from zero, and the
// composition of its transitions.  A product of one-hot-column-times-diagonal matrices is again
// one: column j of the composed map has weight f_w[j] in row f_pi[j], and one more step k gives
// f_pi <- dict[k][f_pi], f_w <- f_w * d_t[f_pi].
template <int N>
__global__ void __launch_bounds__(NT) pdssm_fwd_summary_kernel(PdArgs p) {
    constexpr int SEQ = NT / N, TT = 16;
    __shared__ __align__(16) float sd[2][TT * NT];
    __shared__ __align__(16) float sb[2][TT * NT];
    __shared__ __align__(16) int ssel[2][TT * SEQ];
    __shared__ float sv[NT];
    __shared__ unsigned char s_start[KMAX * (N + 1)];
    __shared__ unsigned char s_src[KMAX * N];
    __shared__ unsigned char s_dict[KMAX * N];
    const int tid = threadIdx.x, j = tid % N, sq = tid / N;
    const int b = blockIdx.y, e0 = blockIdx.x * SEQ, e = e0 + sq, seg = blockIdx.z;
    const bool ev = e < p.H;
    const size_t total = (size_t)p.B * p.L * p.H;
    build_lists<N>(p.dict, p.K, s_start, s_src, tid, p.status);
    for (int i = tid; i < p.K * N; i += NT) s_dict[i] = (unsigned char)dict_row<N>(p.dict, i, p.status);
    const int t_begin = seg * p.seg_len, t_end = min(p.L, t_begin + p.seg_len);
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    auto row0 = [&](int t) { return ((size_t)b * p.L + t) * p.H + e0; };
    const size_t rstride = (size_t)p.H * N;
    auto issue = [&](int jt, int st) {
        const size_t o = row0(t_begin + jt * TT);
        tile_rows<TT>(sd[st], p.d, o * N, rstride, total * N, tid);
        tile_rows<TT>(sb[st], p.bt, o * N, rstride, total * N, tid);
        tile_sel<TT, SEQ>(ssel[st], p.sel, o, p.H, total, tid);
        cp_async_commit();
    };
    __syncthreads();
    float h = 0.0f, w = 1.0f;
    int pi = j;
    if (ntiles > 0) issue(0, 0);
    for (int jt = 0; jt < ntiles; ++jt) {
        const int st = jt & 1;
        if (jt + 1 < ntiles) {
            issue(jt + 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int rows = min(TT, t_end - (t_begin + jt * TT));
        for (int r = 0; r < rows; ++r) {
            const int k = min(max(ssel[st][r * SEQ + sq], 0), p.K - 1);
            sv[tid] = sd[st][r * NT + tid] * h;
            __syncwarp();
            float acc = sb[st][r * NT + tid];
            const int q1 = s_start[k * (N + 1) + j + 1];
            for (int q = s_start[k * (N + 1) + j]; q < q1; ++q) acc += sv[sq * N + s_src[k * N + q]];
            h = acc;
            w *= sd[st][r * NT + sq * N + pi];
            pi = s_dict[k * N + pi];
            __syncwarp();
        }
        __syncthreads();
    }
    if (ev) {
        const size_t o = (((size_t)b * p.H + e) * (p.nseg - 1) + seg) * N + j;
        p.f_pi[o] = pi;
        p.f_w[o] = w;
        p.f_s[o] = h;
    }
}

// Phase B of the forward: h_in[0] = h0 (or zero), h_in[s+1] = M_s h_in[s] + S_s, one N-lane group
// per (batch, head); the scatter of M_s is a fixed-order loop over the group's lanes.
template <int N>
__global__ void __launch_bounds__(NT) pdssm_carry_fwd_kernel(PdArgs p) {
    const int tid = threadIdx.x, j = tid % N;
    const int64_t be = ((int64_t)blockIdx.x * NT + tid) / N;  // (b, e) row
    const bool ok = be < (int64_t)p.B * p.H;
    const int lane = tid & 31, base = lane & ~(N - 1);
    float h = (ok && p.h0) ? p.h0[be * N + j] : 0.0f;
    for (int s = 0; s < p.nseg; ++s) {
        if (ok) p.hin[(be * p.nseg + s) * N + j] = h;
        if (s == p.nseg - 1) break;
        const size_t o = ((size_t)be * (p.nseg - 1) + s) * N + j;
        const int pi = ok ? p.f_pi[o] : 0;
        const float x = ok ? p.f_w[o] * h : 0.0f;
        float acc = ok ? p.f_s[o] : 0.0f;
        for (int jj = 0; jj < N; ++jj) {
            const int pj = __shfl_sync(0xffffffffu, pi, base + jj);
            const float xj = __shfl_sync(0xffffffffu, x, base + jj);
            if (pj == j) acc += xj;
        }
        h = acc;
    }
}

// Phase A of the backward (segments 1..nseg-1): the adjoint sweep of the segment from zero, and
// the composition of its transposed transitions, a gather map: (G x)_j = b_v[j] x[b_rho[j]];
// one more step t (going backwards) gives b_rho <- b_rho[dict[k][j]], b_v <- d_t[j] b_v[dict[k][j]].
template <int N>
__global__ void __launch_bounds__(NT) pdssm_bwd_summary_kernel(PdArgs p) {
    constexpr int SEQ = NT / N, TT = 8;
    __shared__ __align__(16) float sg[2][TT * NT];
    __shared__ __align__(16) float sd[2][TT * NT];
    __shared__ __align__(16) int ssel[2][TT * SEQ];
    __shared__ float sv[NT];
    __shared__ unsigned char s_dict[KMAX * N];
    const int tid = threadIdx.x, j = tid % N, sq = tid / N;
    const int b = blockIdx.y, e0 = blockIdx.x * SEQ, e = e0 + sq, seg = blockIdx.z + 1;
    const bool ev = e < p.H;
    const int lane = tid & 31, gbase = lane & ~(N - 1);
    const size_t total = (size_t)p.B * p.L * p.H;
    for (int i = tid; i < p.K * N; i += NT) s_dict[i] = (unsigned char)dict_row<N>(p.dict, i, p.status);
    const int t_begin = seg * p.seg_len, t_end = min(p.L, t_begin + p.seg_len);
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    auto row0 = [&](int t) { return ((size_t)b * p.L + t) * p.H + e0; };
    const size_t rstride = (size_t)p.H * N;
    auto issue = [&](int jt, int st) {
        const size_t o = row0(t_begin + jt * TT);
        tile_rows<TT>(sg[st], p.g, o * N, rstride, total * N, tid);
        tile_rows<TT>(sd[st], p.d, o * N, rstride, total * N, tid);
        tile_sel<TT, SEQ>(ssel[st], p.sel, o, p.H, total, tid);
        cp_async_commit();
    };
    __syncthreads();
    float w = 0.0f, v = 1.0f;
    int rho = j;
    if (ntiles > 0) issue(ntiles - 1, (ntiles - 1) & 1);
    for (int jt = ntiles - 1; jt >= 0; --jt) {
        const int st = jt & 1;
        if (jt > 0) {
            issue(jt - 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int rows = min(TT, t_end - (t_begin + jt * TT));
        for (int r = rows - 1; r >= 0; --r) {
            const int k = min(max(ssel[st][r * SEQ + sq], 0), p.K - 1);
            const float dj = sd[st][r * NT + tid];
            const float mu = sg[st][r * NT + tid] + w;
            sv[tid] = mu;
            __syncwarp();
            const int src = s_dict[k * N + j];
            w = dj * sv[sq * N + src];
            const int rho_n = __shfl_sync(0xffffffffu, rho, gbase + src);
            const float v_n = __shfl_sync(0xffffffffu, v, gbase + src);
            rho = rho_n;
            v = dj * v_n;
            __syncwarp();
        }
        __syncthreads();
    }
    if (ev) {
        const size_t o = (((size_t)b * p.H + e) * (p.nseg - 1) + (seg - 1)) * N + j;
        p.b_rho[o] = rho;
        p.b_v[o] = v;
        p.b_w[o] = w;
    }
}

// Phase B of the backward: w_in[nseg-1] = 0, w_in[s-1] = W_s + G_s w_in[s] (a gather).
template <int N>
__global__ void __launch_bounds__(NT) pdssm_carry_bwd_kernel(PdArgs p) {
    const int tid = threadIdx.x, j = tid % N;
    const int64_t be = ((int64_t)blockIdx.x * NT + tid) / N;
    const bool ok = be < (int64_t)p.B * p.H;
    const int lane = tid & 31, base = lane & ~(N - 1);
    float w = 0.0f;
    for (int s = p.nseg - 1; s >= 0; --s) {
        if (ok) p.win[(be * p.nseg + s) * N + j] = w;
        if (s == 0) break;
        const size_t o = ((size_t)be * (p.nseg - 1) + (s - 1)) * N + j;
        const int rho = ok ? p.b_rho[o] : j;
        const float g = __shfl_sync(0xffffffffu, w, base + rho);
        w = ok ? fmaf(p.b_v[o], g, p.b_w[o]) : 0.0f;
    }
}

// Straight-through score gradient, one thread per (b, t, e): c_k = <mu_t, P_k D_t h_{t-1}> with
// mu_t = dbt (written by the backward scan), then dscores = p (c - <p, c>) / tau.
template <int N>
__global__ void __launch_bounds__(NT) pdssm_dscores_kernel(PdArgs p) {
    __shared__ float smu[NT][N + 1];
    __shared__ unsigned char s_dict[KMAX * N];
    const int tid = threadIdx.x;
    for (int i = tid; i < p.K * N; i += NT) s_dict[i] = (unsigned char)dict_row<N>(p.dict, i, p.status);
    const int64_t n = (int64_t)p.B * p.L * p.H;
    const int64_t i = (int64_t)blockIdx.x * NT + tid;
    const bool ok = i < n;
    float x[N];  // d_t[j] h_{t-1}[j]
    if (ok) {
        const int64_t t = (i / p.H) % p.L;
        const float* mu = p.dbt + i * N;
        const float* dr = p.d + i * N;
        const float* hp = t > 0 ? p.h + (i - p.H) * N : nullptr;
        const float* h0 = p.h0 ? p.h0 + ((i / ((int64_t)p.L * p.H)) * p.H + i % p.H) * N : nullptr;
#pragma unroll
        for (int jj = 0; jj < N; jj += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(mu + jj);
            const float4 d4 = *reinterpret_cast<const float4*>(dr + jj);
            float4 h4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (hp)
                h4 = *reinterpret_cast<const float4*>(hp + jj);
            else if (h0)
                h4 = *reinterpret_cast<const float4*>(h0 + jj);
            smu[tid][jj] = m4.x; smu[tid][jj + 1] = m4.y; smu[tid][jj + 2] = m4.z; smu[tid][jj + 3] = m4.w;
            x[jj] = d4.x * h4.x; x[jj + 1] = d4.y * h4.y; x[jj + 2] = d4.z * h4.z; x[jj + 3] = d4.w * h4.w;
        }
    }
    __syncthreads();
    if (!ok) return;
    const float* sc = p.scores + i * p.K;
    float mx = sc[0];
    for (int k = 1; k < p.K; ++k) mx = fmaxf(mx, sc[k]);
    const float it = 1.0f / p.tau;
    float z = 0.0f, pc = 0.0f;
    for (int k = 0; k < p.K; ++k) {
        float ck = 0.0f;
#pragma unroll
        for (int jj = 0; jj < N; ++jj) ck = fmaf(smu[tid][s_dict[k * N + jj]], x[jj], ck);
        const float pk = expf((sc[k] - mx) * it);
        z += pk;
        pc = fmaf(pk, ck, pc);
        p.dscores[i * p.K + k] = ck;  // c_k for now
    }
    const float rz = 1.0f / z, mean = pc * rz;
    for (int k = 0; k < p.K; ++k) {
        const float pk = expf((sc[k] - mx) * it) * rz;
        p.dscores[i * p.K + k] = pk * (p.dscores[i * p.K + k] - mean) * it;
    }
}

template <int N>
cudaError_t fwd_impl(const PdArgs& a, cudaStream_t st) {
    const int64_t n = (int64_t)a.B * a.L * a.H;
    pdssm_select_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int seq = NT / N;
    const unsigned gx = (unsigned)((a.H + seq - 1) / seq);
    if (a.nseg > 1) {
        pdssm_fwd_summary_kernel<N><<<dim3(gx, a.B, a.nseg - 1), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t groups = (int64_t)a.B * a.H * N;
        pdssm_carry_fwd_kernel<N><<<(unsigned)((groups + NT - 1) / NT), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    pdssm_fwd_kernel<N><<<dim3(gx, a.B, a.nseg), NT, 0, st>>>(a);
    return cudaGetLastError();
}

template <int N>
cudaError_t bwd_impl(const PdArgs& a, cudaStream_t st) {
    const int seq = NT / N;
    const unsigned gx = (unsigned)((a.H + seq - 1) / seq);
    cudaError_t e;
    if (a.nseg > 1) {
        pdssm_bwd_summary_kernel<N><<<dim3(gx, a.B, a.nseg - 1), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t groups = (int64_t)a.B * a.H * N;
        pdssm_carry_bwd_kernel<N><<<(unsigned)((groups + NT - 1) / NT), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    pdssm_bwd_kernel<N><<<dim3(gx, a.B, a.nseg), NT, 0, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)a.B * a.L * a.H;
    pdssm_dscores_kernel<N><<<(unsigned)((n + NT - 1) / NT), NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pdssm_fwd(const PdArgs& a, cudaStream_t st) {
    switch (a.N) {
        case 4: return fwd_impl<4>(a, st);
        case 8: return fwd_impl<8>(a, st);
        case 16: return fwd_impl<16>(a, st);
        default: return fwd_impl<32>(a, st);
    }
}

cudaError_t launch_pdssm_bwd(const PdArgs& a, cudaStream_t st) {
    switch (a.N) {
        case 4: return bwd_impl<4>(a, st);
        case 8: return bwd_impl<8>(a, st);
        case 16: return bwd_impl<16>(a, st);
        default: return bwd_impl<32>(a, st);
    }
}

}  // namespace ssm
