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
// row, each warp 32 / N of them, lane j of each N-lane group owning state j; one step of a warp
// reads and writes 128 contiguous bytes per array.  Every warp runs its own pipeline: tiles of 16
// steps through a three-stage cp.async ring, no barrier with the other warps inside the loop.
//   forward:  per tile, the argmax of the staged scores (one lane per (step, head)), then the
//             scan; the scatter of P_k (several columns may land on one row) is a gather over the
//             row's in-list, padded to the dictionary's largest in-degree D, through register
//             shuffles within the N-lane group: one packed word of source lanes per (k, row).
//   backward: per tile, the reverse scan (the transposed gather is one shuffle per step), with
//             mu and x = d h_{t-1} left in shared memory; then the score gradient, one lane per
//             (step, head), from them and the staged scores.
// When the (batch, head-group) CTAs cannot fill the GPU the sequence is cut into time segments
// (local scans with composed maps, a carry, a rescan).  When a tile's scores would not fit the
// staging budget (K * heads-per-CTA > 256) the argmax and the score gradient run as separate
// kernels parallel over (b, t, e).
#include "real_common.cuh"

namespace ssm {
namespace {

using real::cp_async_commit;
using real::cp_async_wait;
using real::kFull;

constexpr int NT = kPdThreads;
constexpr int KMAX = 32;      // dictionary size limit (validated on the host)
constexpr int TT = 16;        // steps per staged tile
constexpr int STAGES = 3;     // cp.async ring depth
constexpr int DPAD = 7;       // padded in-degrees 1..DPAD use the packed-word gather
constexpr int SCORE_ROW_MAX = 256;  // K * heads-per-CTA staged per step (fused select / dscores)

// Value of lane (group base + (src mod N)) of this lane's N-lane group: __shfl_sync with width N
// reads the source lane modulo the width, so a packed word shifted right by 8 m selects its m-th
// byte without masking.
template <int N>
__device__ __forceinline__ float grp_shfl(float v, unsigned src) {
    return __shfl_sync(kFull, v, (int)src, N);
}

__host__ __device__ constexpr int align16i(int x) { return (x + 15) & ~15; }

// sel[b,t,e] = argmax_k scores[b,t,e,k], lowest index on ties.
__device__ __forceinline__ int argmax_k(const float* sc, int K) {
    int kb = 0;
    float best = sc[0];
    for (int k = 1; k < K; ++k) {
        const float v = sc[k];
        if (v > best) {
            best = v;
            kb = k;
        }
    }
    return kb;
}

__global__ void pdssm_select_kernel(PdArgs p) {
    const int64_t n = (int64_t)p.B * p.L * p.H;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    p.sel[i] = argmax_k(p.scores + i * p.K, p.K);
}

// Copy the rows t0 .. t0+R-1 of one CTA (NT consecutive floats per row, row stride H*N floats)
// of a [B, L, H, N] array into dst[R][NT], 16 bytes per piece; pieces past the array end read as
// zero (rows past L of a batch row are never used).
template <int R>
__device__ __forceinline__ void tile_rows(float* dst, const float* src, size_t first, size_t stride,
                                          size_t total, int tid) {
    constexpr int PR = NT / 4;  // pieces per row
#pragma unroll
    for (int q = tid; q < R * PR; q += NT) {
        const int r = q / PR, c = q - r * PR;
        const size_t e = first + (size_t)r * stride + 4 * c;
        const bool ok = e + 4 <= total;
        real::cp_async16(dst + r * NT + 4 * c, ok ? src + e : src, ok);
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
// ascending j, at src[k*N + start[k*(N+1) + i] ...].  Also the dictionary itself as bytes.
template <int N>
__device__ __forceinline__ void build_lists(const int32_t* dict, int K, unsigned char* start,
                                            unsigned char* src, unsigned char* sdict, int tid,
                                            unsigned* status) {
    for (int k = tid; k < K; k += NT) {
        int cnt[N];
#pragma unroll
        for (int i = 0; i < N; ++i) cnt[i] = 0;
        for (int j = 0; j < N; ++j) {
            const int i = dict_row<N>(dict, k * N + j, status);
            sdict[k * N + j] = (unsigned char)i;
            ++cnt[i];
        }
        int acc = 0;
#pragma unroll
        for (int i = 0; i < N; ++i) {
            start[k * (N + 1) + i] = (unsigned char)acc;
            acc += cnt[i];
            cnt[i] = start[k * (N + 1) + i];
        }
        start[k * (N + 1) + N] = (unsigned char)acc;
        for (int j = 0; j < N; ++j) src[k * N + cnt[sdict[k * N + j]]++] = (unsigned char)j;
    }
}

// Largest in-degree D over all (k, row), and, when D <= DPAD, the packed gather words: for
// (k, row i) bytes 0..6 hold the source columns in ascending order (unused bytes: i itself) and
// byte 7 the count.  Call after build_lists and a barrier; ends with a barrier.
template <int N>
__device__ __forceinline__ int build_words(const unsigned char* start, const unsigned char* src,
                                           int K, uint2* words, int* s_deg, int tid) {
    if (tid == 0) *s_deg = 0;
    __syncthreads();
    for (int q = tid; q < K * N; q += NT) {
        const int k = q / N, i = q - k * N;
        atomicMax(s_deg, start[k * (N + 1) + i + 1] - start[k * (N + 1) + i]);
    }
    __syncthreads();
    const int D = *s_deg;
    if (D <= DPAD) {
        for (int q = tid; q < K * N; q += NT) {
            const int k = q / N, i = q - k * N;
            const int a = start[k * (N + 1) + i], c = start[k * (N + 1) + i + 1] - a;
            unsigned w[2] = {0u, 0u};
            for (int m = 0; m < 7; ++m) {
                const unsigned s = m < c ? src[k * N + a + m] : (unsigned)i;
                w[m >> 2] |= s << (8 * (m & 3));
            }
            w[1] |= (unsigned)c << 24;
            words[q] = make_uint2(w[0], w[1]);
        }
    }
    __syncthreads();
    return D;
}

// acc + sum over the in-list of this lane's row of x (read from the source lanes): D padded
// entries from the packed word (DW > 0), or the plain lists up to the runtime bound Dm (DW == 0).
template <int N, int DW>
__device__ __forceinline__ float gather_add(float acc, float x, int k, int j, const uint2* words,
                                            const unsigned char* start, const unsigned char* src,
                                            int Dm) {
    if constexpr (DW > 0) {
        // the D values are independent: zero the padding, then a pairwise tree (depth log2 D
        // instead of a chain of D dependent adds)
        const uint2 w = words[k * N + j];
        const int c = (int)(w.y >> 24);
        float v[DW];
#pragma unroll
        for (int m = 0; m < DW; ++m) {
            const unsigned s = m < 4 ? w.x >> (8 * m) : w.y >> (8 * (m - 4));
            const float u = grp_shfl<N>(x, s);
            v[m] = m < c ? u : 0.0f;
        }
#pragma unroll
        for (int span = 1; span < DW; span *= 2) {
#pragma unroll
            for (int m = 0; m + span < DW; m += 2 * span) v[m] += v[m + span];
        }
        acc += v[0];
    } else {
        const int a = start[k * (N + 1) + j], c = start[k * (N + 1) + j + 1] - a;
        for (int m = 0; m < Dm; ++m) {
            const unsigned s = m < c ? src[k * N + a + m] : (unsigned)j;
            const float v = grp_shfl<N>(x, s);
            if (m < c) acc += v;
        }
    }
    return acc;
}

// ------------------------------------------------------------------------------------------------
// Per-warp pipelines.  A warp owns SPW = 32 / N consecutive heads (lane = head c, state j).  Its
// tiles (TT steps x 32 floats per array: 128 contiguous bytes per step) go through its own
// three-stage cp.async ring and its (step, head) entries through its own lanes, so the warps of a
// CTA never wait for one another inside the sequence loop (a warp in its latency-bound scan runs
// beside one in its score-gradient phase); only the dictionary tables are shared.

// TT rows of 32 floats (row stride `stride`) into dst[TT][32], rows from `r0` on; 16-byte pieces,
// zero past `total`.
__device__ __forceinline__ void warp_rows(float* dst, const float* src, size_t first, size_t stride,
                                          size_t total, int r0, int lane) {
#pragma unroll
    for (int q = lane + 8 * r0; q < TT * 8; q += 32) {
        const int r = q >> 3, c4 = q & 7;
        const size_t e = first + (size_t)(r - r0) * stride + 4 * c4;
        const bool ok = e + 4 <= total;
        real::cp_async16(dst + r * 32 + 4 * c4, ok ? src + e : src, ok);
    }
}

// 4-byte pieces: TT rows of `spw` entries of `w` elements each (row stride `stride`), entry
// (r, c) to dst[(r * spw + c) * ds ...]; zero past `total`.
__device__ __forceinline__ void warp_entries(void* dst, const void* src, size_t first, size_t stride,
                                             int spw, int w, int ds, size_t total, int lane) {
    const float* s = static_cast<const float*>(src);
    float* d = static_cast<float*>(dst);
    for (int ent = lane; ent < TT * spw; ent += 32) {
        const int r = ent / spw, c = ent - r * spw;
        const size_t e0 = first + (size_t)r * stride + (size_t)c * w;
        for (int k = 0; k < w; ++k) {
            const size_t e = e0 + k;
            const unsigned sa = (unsigned)__cvta_generic_to_shared(d + ent * ds + k);
            const int n = e < total ? 4 : 0;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(sa),
                         "l"(n ? s + e : s), "r"(n));
        }
    }
}

// Forward shared memory: per warp d, bt [STAGES][TT][32], the staged scores [STAGES][TT*SPW][K+1]
// (odd entry stride: the entry-per-lane reads hit distinct banks) and the tile's selection; then
// the CTA's dictionary tables.
struct FwdLayout {
    int sd, sb, ssc, ssel, warp;
    int words, start, src, dict, deg, total;
};

__host__ __device__ inline FwdLayout fwd_layout(int N, int K, bool fused) {
    const int spw = 32 / N;
    FwdLayout l;
    int o = 0;
    l.sd = o;   o += STAGES * TT * 32 * 4;
    l.sb = o;   o += STAGES * TT * 32 * 4;
    l.ssc = o;  o += fused ? align16i(STAGES * TT * spw * (K + 1) * 4) : 0;
    l.ssel = o; o += align16i(TT * spw * 4);
    l.warp = o;
    o *= NT / 32;
    l.words = o; o += align16i(K * N * 8);
    l.start = o; o += align16i(K * (N + 1));
    l.src = o;   o += align16i(K * N);
    l.dict = o;  o += align16i(K * N);
    l.deg = o;   o += 16;
    l.total = o;
    return l;
}

struct PdTables {
    const uint2* words;
    const unsigned char* start;
    const unsigned char* src;
    const unsigned char* dict;
};

// One warp's heads over one segment: SUMMARY == false scans from the segment's entering state and
// writes h (and sel, when the select is fused); SUMMARY == true scans from zero and composes the
// segment's transitions (phase A of the segmented forward: a product of one-hot-column-times-
// diagonal matrices is again one; column j of the composed map has weight w in row pi, and one
// more step k gives pi <- dict[k][pi], w <- w * d_t[pi]).
template <int N, int DW, bool SUMMARY>
__device__ __forceinline__ void fwd_body(const PdArgs& p, unsigned char* wsm, const FwdLayout& l,
                                         const PdTables& tb, bool fused, int Dm) {
    constexpr int SPW = 32 / N;
    const int lane = threadIdx.x & 31, c = lane / N, j = lane % N;
    const int b = blockIdx.y, e0 = blockIdx.x * (NT / N) + (threadIdx.x >> 5) * SPW, e = e0 + c;
    const bool ev = e < p.H;
    float* sd = reinterpret_cast<float*>(wsm + l.sd);
    float* sb = reinterpret_cast<float*>(wsm + l.sb);
    float* ssc = reinterpret_cast<float*>(wsm + l.ssc);
    int* ssel = reinterpret_cast<int*>(wsm + l.ssel);
    const int K = p.K, KP = K + 1;
    const size_t total = (size_t)p.B * p.L * p.H;  // (b, t, e) rows
    const int seg = blockIdx.z;
    const int t_begin = seg * p.seg_len, t_end = min(p.L, t_begin + p.seg_len);
    float h = 0.0f, w = 1.0f;
    int pi = j;
    if (!SUMMARY && ev) {
        if (p.nseg > 1)
            h = p.hin[(((size_t)b * p.H + e) * p.nseg + seg) * N + j];
        else if (p.h0)
            h = p.h0[((size_t)b * p.H + e) * N + j];
    }
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    auto row0 = [&](int t) { return ((size_t)b * p.L + t) * p.H + e0; };  // the warp's first row
    const size_t rstride = (size_t)p.H * N;
    auto issue = [&](int jt) {
        if (jt < ntiles) {
            const int st = jt % STAGES;
            const size_t o = row0(t_begin + jt * TT);
            warp_rows(sd + st * TT * 32, p.d, o * N, rstride, total * N, 0, lane);
            warp_rows(sb + st * TT * 32, p.bt, o * N, rstride, total * N, 0, lane);
            if (fused)
                warp_entries(ssc + st * TT * SPW * KP, p.scores, o * K, (size_t)p.H * K, SPW, K, KP,
                             total * K, lane);
        }
        cp_async_commit();
    };
    issue(0);
    issue(1);
    for (int jt = 0; jt < ntiles; ++jt) {
        const int st = jt % STAGES;
        cp_async_wait<STAGES - 2>();
        __syncwarp();  // tile jt is in for every lane; every lane is done with tile jt-1
        issue(jt + 2);
        const int t0 = t_begin + jt * TT, rows = min(TT, t_end - t0);
        for (int ent = lane; ent < TT * SPW; ent += 32) {
            const int r = ent / SPW, cc = ent - r * SPW;
            int kb = 0;
            if (r < rows && e0 + cc < p.H) {
                if (fused) {
                    kb = argmax_k(ssc + st * TT * SPW * KP + ent * KP, K);
                    if (!SUMMARY) p.sel[row0(t0 + r) + cc] = kb;
                } else {
                    kb = min(max(p.sel[row0(t0 + r) + cc], 0), K - 1);
                }
            }
            ssel[ent] = kb;
        }
        __syncwarp();
        const float* sdt = sd + st * TT * 32;
        const float* sbt = sb + st * TT * 32;
        float* hout = p.h + row0(t0) * N + lane;
        const unsigned rs32 = (unsigned)rstride;  // 16 * H * N < 2^32 (heads <= 2^21)
#pragma unroll 4
        for (int r = 0; r < rows; ++r) {
            const int k = ssel[r * SPW + c];
            const float x = sdt[r * 32 + lane] * h;
            h = gather_add<N, DW>(sbt[r * 32 + lane], x, k, j, tb.words, tb.start, tb.src, Dm);
            if constexpr (SUMMARY) {
                w *= sdt[r * 32 + c * N + pi];
                pi = tb.dict[k * N + pi];
            } else if (ev) {
                hout[(unsigned)r * rs32] = h;
            }
        }
    }
    if constexpr (SUMMARY) {
        if (ev) {
            const size_t o = (((size_t)b * p.H + e) * (p.nseg - 1) + seg) * N + j;
            p.f_pi[o] = pi;
            p.f_w[o] = w;
            p.f_s[o] = h;
        }
    } else {
        if (ev && !isfinite(h)) flag_status(p.status, kStatusNonFinite);
    }
}

template <int N, bool SUMMARY>
__global__ void __launch_bounds__(NT) pdssm_fwd_kernel(PdArgs p) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int SEQ = NT / N;
    const bool fused = SEQ * p.K <= SCORE_ROW_MAX;
    const FwdLayout l = fwd_layout(N, p.K, fused);
    unsigned char* start = smem + l.start;
    unsigned char* src = smem + l.src;
    unsigned char* dict = smem + l.dict;
    uint2* words = reinterpret_cast<uint2*>(smem + l.words);
    const int tid = threadIdx.x;
    build_lists<N>(p.dict, p.K, start, src, dict, tid, p.status);
    __syncthreads();
    const int D = build_words<N>(start, src, p.K, words, reinterpret_cast<int*>(smem + l.deg), tid);
    const PdTables tb = {words, start, src, dict};
    unsigned char* wsm = smem + (tid >> 5) * l.warp;
    if constexpr (SUMMARY) {
        fwd_body<N, 0, true>(p, wsm, l, tb, fused, D);
    } else {
        switch (D) {
            case 1: fwd_body<N, 1, false>(p, wsm, l, tb, fused, D); break;
            case 2: fwd_body<N, 2, false>(p, wsm, l, tb, fused, D); break;
            case 3: fwd_body<N, 3, false>(p, wsm, l, tb, fused, D); break;
            case 4: fwd_body<N, 4, false>(p, wsm, l, tb, fused, D); break;
            case 5: fwd_body<N, 5, false>(p, wsm, l, tb, fused, D); break;
            case 6: fwd_body<N, 6, false>(p, wsm, l, tb, fused, D); break;
            case 7: fwd_body<N, 7, false>(p, wsm, l, tb, fused, D); break;
            default: fwd_body<N, 0, false>(p, wsm, l, tb, fused, D); break;
        }
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
            const int pj = __shfl_sync(kFull, pi, base + jj);
            const float xj = __shfl_sync(kFull, x, base + jj);
            if (pj == j) acc += xj;
        }
        h = acc;
    }
}

// ------------------------------------------------------------------------------------------------
// Backward: warp-specialised.  A CTA holds two (scan, score-gradient) warp pairs.  The scan warp
// of a pair runs the reverse recurrence over its 32 / N heads (tiles through its own two-stage
// cp.async ring) and leaves mu and x = d h_{t-1} of each tile in one of two shared buffers; the
// score-gradient warp takes the tile from there (one lane per (step, head) entry, the scores
// through its own ring) while the scan warp goes on with the next tile.  The two hand the buffers
// over with named barriers (FULL: written, EMPTY: read; the sequence of barrier operations of
// both roles is model-checked on the host by tests/test_barrier_protocol.py).  The latency-bound
// scan and the arithmetic-bound score gradient so run side by side instead of in turn.
//
// Shared memory per scan warp: g, d, h_{t-1} [2][TT][32] floats and sel [2][TT*SPW]; per pair:
// mu and x [2 buffers][TT][RS] with RS = SPW*(N+1) = 32 + SPW (state i of entry (r, c) at
// r*RS + c*(N+1) + i: a pass of the score gradient gives lane L the entry divmod(L + 32 pass, SPW)
// and reads one dictionary offset i for all lanes, and the 32 addresses fall in 32 distinct banks
// for every N), the scores [2][TT*SPW][K+1] (odd entry stride) and each lane's c_k [32][K+1];
// then the dictionary.
constexpr int BW_STAGES = 2;
constexpr int BW_PAIRS = 2;

struct BwdLayout {
    int prod, pair;                    // region bytes: per scan warp, per pair
    int pg, pd, php, psel;             // offsets within a scan-warp region
    int amu, ax, asc, acc;             // offsets within a pair region
    int dict, total;
};

__host__ __device__ inline BwdLayout bwd_layout(int N, int K, bool fused) {
    const int spw = 32 / N, rs = spw * (N + 1), kp = K + 1;
    BwdLayout l;
    int o = 0;
    l.pg = o;   o += BW_STAGES * TT * 32 * 4;
    l.pd = o;   o += BW_STAGES * TT * 32 * 4;
    l.php = o;  o += BW_STAGES * TT * 32 * 4;
    l.psel = o; o += align16i(BW_STAGES * TT * spw * 4);
    l.prod = o;
    o = 0;
    l.amu = o;  o += fused ? align16i(2 * TT * rs * 4) : 0;
    l.ax = o;   o += fused ? align16i(2 * TT * rs * 4) : 0;
    l.asc = o;  o += fused ? align16i(2 * TT * spw * kp * 4) : 0;
    l.acc = o;  o += fused ? align16i(32 * kp * 4) : 0;
    l.pair = o;
    l.dict = BW_PAIRS * (l.prod + l.pair);
    l.total = l.dict + align16i(K * N);
    return l;
}

__device__ __forceinline__ void named_sync(int id) {
    asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory");
}
__device__ __forceinline__ void named_arrive(int id) {
    asm volatile("bar.arrive %0, 64;\n" ::"r"(id) : "memory");
}

template <int N>
__global__ void __launch_bounds__(NT) pdssm_bwd_kernel(PdArgs p) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int SPW = 32 / N, RS = SPW * (N + 1);
    const int K = p.K, KP = K + 1;
    const bool fused = (NT / N) * K <= SCORE_ROW_MAX;
    const BwdLayout l = bwd_layout(N, K, fused);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pair = warp & 1;                // scan warp `pair`, score warp `pair + 2`
    const bool scan_role = warp < BW_PAIRS;
    unsigned char* sdict = smem + l.dict;
    unsigned char* pr = smem + pair * l.prod;
    unsigned char* pa = smem + BW_PAIRS * l.prod + pair * l.pair;
    float* smu = reinterpret_cast<float*>(pa + l.amu);  // [2][TT][RS]
    float* sx = reinterpret_cast<float*>(pa + l.ax);
    const int c = lane / N, j = lane % N;
    const int b = blockIdx.y, e0 = blockIdx.x * (BW_PAIRS * SPW) + pair * SPW, e = e0 + c;
    const bool ev = e < p.H;
    const size_t total = (size_t)p.B * p.L * p.H;
    for (int i = tid; i < K * N; i += NT) sdict[i] = (unsigned char)dict_row<N>(p.dict, i, p.status);
    const int seg = blockIdx.z;
    const int t_begin = seg * p.seg_len, t_end = min(p.L, t_begin + p.seg_len);
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    auto row0 = [&](int t) { return ((size_t)b * p.L + t) * p.H + e0; };  // the pair's first row
    const size_t rstride = (size_t)p.H * N;
    const int FULL = 1 + 4 * pair, EMPTY = 3 + 4 * pair;  // + buffer index
    __syncthreads();  // dictionary

    if (scan_role) {
        float* sg = reinterpret_cast<float*>(pr + l.pg);
        float* sd = reinterpret_cast<float*>(pr + l.pd);
        float* shp = reinterpret_cast<float*>(pr + l.php);  // h_{t-1} of the tile's steps
        int* ssel = reinterpret_cast<int*>(pr + l.psel);
        auto issue = [&](int jt) {
            if (jt >= 0) {
                const int st = jt % BW_STAGES;
                const int t0 = t_begin + jt * TT;
                const size_t o = row0(t0);
                float* hp = shp + st * TT * 32;
                warp_rows(sg + st * TT * 32, p.g, o * N, rstride, total * N, 0, lane);
                warp_rows(sd + st * TT * 32, p.d, o * N, rstride, total * N, 0, lane);
                warp_entries(ssel + st * TT * SPW, p.sel, o, p.H, SPW, 1, 1, total, lane);
                if (t0 > 0) {
                    warp_rows(hp, p.h, (o - p.H) * N, rstride, total * N, 0, lane);
                } else {  // row 0 is h_{-1} = h0 (or zero), rows 1.. the trajectory
                    warp_rows(hp, p.h, o * N, rstride, total * N, 1, lane);
                    if (p.h0) {
                        const size_t bh = (size_t)p.B * p.H * N, f = ((size_t)b * p.H + e0) * N;
                        if (lane < 8) {
                            const size_t q = f + 4 * lane;
                            real::cp_async16(hp + 4 * lane, q + 4 <= bh ? p.h0 + q : p.h0, q + 4 <= bh);
                        }
                    } else {
                        hp[lane] = 0.0f;
                    }
                }
            }
            cp_async_commit();
        };
        const unsigned rs32 = (unsigned)rstride;
        float w = 0.0f;  // A_{t+1}^T mu_{t+1}: from the carry (or later segment), zero at the end
        if (ev && seg < p.nseg - 1) w = p.win[(((size_t)b * p.H + e) * p.nseg + seg) * N + j];
        issue(ntiles - 1);
        for (int i = 0; i < ntiles; ++i) {
            const int jt = ntiles - 1 - i, st = jt % BW_STAGES, buf = i & 1;
            cp_async_wait<0>();
            __syncwarp();  // tile jt is in for every lane; every lane is done with tile jt+1
            issue(jt - 1);
            const int t0 = t_begin + jt * TT, rows = min(TT, t_end - t0);
            const float* sgt = sg + st * TT * 32;
            const float* sdt = sd + st * TT * 32;
            const float* shpt = shp + st * TT * 32;
            const int* sst = ssel + st * TT * SPW;
            float* mub = smu + buf * TT * RS;
            float* xb = sx + buf * TT * RS;
            float* dbt = p.dbt + row0(t0) * N + lane;
            float* dd = p.dd + row0(t0) * N + lane;
            if (fused) named_sync(EMPTY + buf);  // the score warp is done with this buffer
#pragma unroll 4
            for (int r = rows - 1; r >= 0; --r) {
                const int k = min(max(sst[r * SPW + c], 0), K - 1);
                const float mu = sgt[r * 32 + lane] + w;
                const float m = grp_shfl<N>(mu, sdict[k * N + j]);  // mu[dict[k][j]]
                const float hp = shpt[r * 32 + lane], dj = sdt[r * 32 + lane];
                if (ev) {  // 32-bit step offsets: 16 * H * N < 2^32 (heads <= 2^21)
                    dbt[(unsigned)r * rs32] = mu;
                    dd[(unsigned)r * rs32] = m * hp;
                }
                if (fused) {
                    mub[r * RS + lane + c] = mu;  // r*RS + c*(N+1) + j
                    xb[r * RS + lane + c] = dj * hp;
                }
                w = dj * m;
            }
            if (fused) named_arrive(FULL + buf);
        }
        if (fused) {  // balance the score warp's last two releases
            named_sync(EMPTY + 0);
            named_sync(EMPTY + 1);
        }
        if (ev) {
            if (p.dh0 && seg == 0) p.dh0[((size_t)b * p.H + e) * N + j] = w;
            if (!isfinite(w)) flag_status(p.status, kStatusNonFinite);
        }
        return;
    }

    if (!fused) return;
    // score-gradient warp: straight-through gradient of the pair's (step, head) entries
    float* ssc = reinterpret_cast<float*>(pa + l.asc);       // [2][TT*SPW][KP]
    float* scc = reinterpret_cast<float*>(pa + l.acc) + lane * KP;
    auto issue_sc = [&](int jt, int st) {
        if (jt >= 0) {
            const size_t o = row0(t_begin + jt * TT);
            warp_entries(ssc + st * TT * SPW * KP, p.scores, o * K, (size_t)p.H * K, SPW, K, KP,
                         total * K, lane);
        }
        cp_async_commit();
    };
    const float itl = kLog2e / p.tau, it = 1.0f / p.tau;
    issue_sc(ntiles - 1, 0);
    named_arrive(EMPTY + 0);  // both buffers start empty
    named_arrive(EMPTY + 1);
    for (int i = 0; i < ntiles; ++i) {
        const int jt = ntiles - 1 - i, buf = i & 1;
        __syncwarp();  // every lane is done with the scores stage of tile jt+1
        issue_sc(jt - 1, (i + 1) & 1);
        cp_async_wait<1>();
        __syncwarp();
        const int t0 = t_begin + jt * TT, rows = min(TT, t_end - t0);
        const float* sct = ssc + buf * TT * SPW * KP;
        const float* mub = smu + buf * TT * RS;
        const float* xb = sx + buf * TT * RS;
        named_sync(FULL + buf);  // the scan warp has written the tile's mu and x
        for (int ent = lane; ent < TT * SPW; ent += 32) {
            const int r = ent / SPW, cc = ent - r * SPW;
            if (r >= rows || e0 + cc >= p.H) continue;
            const float* mur = mub + r * RS + cc * (N + 1);
            const float* xr = xb + r * RS + cc * (N + 1);
            float x[N];
#pragma unroll
            for (int jj = 0; jj < N; ++jj) x[jj] = xr[jj];
            const float* sc = sct + ent * KP;
            float mx = sc[0];
            for (int kk = 1; kk < K; ++kk) mx = fmaxf(mx, sc[kk]);
            const float mxl = mx * itl;
            float z = 0.0f, pc = 0.0f;
            for (int kk = 0; kk < K; ++kk) {
                const unsigned char* dk = sdict + kk * N;
                float c0 = 0.0f, c1 = 0.0f;
#pragma unroll
                for (int jj = 0; jj < N; jj += 2) {
                    c0 = fmaf(mur[dk[jj]], x[jj], c0);
                    c1 = fmaf(mur[dk[jj + 1]], x[jj + 1], c1);
                }
                const float ck = c0 + c1;
                const float pk = ex2_mufu(fmaf(sc[kk], itl, -mxl));  // exp((s_k - max) / tau)
                z += pk;
                pc = fmaf(pk, ck, pc);
                scc[kk] = ck;
            }
            const float rz = 1.0f / z, mean = pc * rz;
            float* out = p.dscores + row0(t0) * K + ((unsigned)r * (unsigned)(p.H * K) + (unsigned)(cc * K));
            for (int kk = 0; kk < K; ++kk) {
                const float pk = ex2_mufu(fmaf(sc[kk], itl, -mxl)) * rz;
                out[kk] = pk * (scc[kk] - mean) * it;
            }
        }
        named_arrive(EMPTY + buf);  // mu and x of this buffer are consumed
    }
}

// The int32 selection of R steps, one (b, t, e) entry per 4-byte piece (segment summaries).
template <int R, int SEQ>
__device__ __forceinline__ void tile_sel(int* dst, const int32_t* src, size_t first, size_t stride,
                                         size_t total, int tid) {
    for (int q = tid; q < R * SEQ; q += NT) {
        const int r = q / SEQ, c = q - r * SEQ;
        const size_t e = first + (size_t)r * stride + c;
        const unsigned sa = (unsigned)__cvta_generic_to_shared(dst + q);
        const int n = e < total ? 4 : 0;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(sa),
                     "l"(n ? src + e : src), "r"(n));
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

// Straight-through score gradient as a kernel of its own (when a tile's scores exceed the staging
// budget), one thread per (b, t, e): c_k = <mu_t, P_k D_t h_{t-1}> with mu_t = dbt (written by the
// backward scan), then dscores = p (c - <p, c>) / tau.
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

template <typename Kern>
cudaError_t launch_dyn(Kern kern, dim3 grid, int bytes, cudaStream_t st, const PdArgs& a) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, NT, bytes, st>>>(a);
    return cudaGetLastError();
}

template <int N>
cudaError_t fwd_impl(const PdArgs& a, cudaStream_t st) {
    constexpr int SEQ = NT / N;
    const bool fused = SEQ * a.K <= SCORE_ROW_MAX;
    cudaError_t e;
    if (!fused) {
        const int64_t n = (int64_t)a.B * a.L * a.H;
        pdssm_select_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const unsigned gx = (unsigned)((a.H + SEQ - 1) / SEQ);
    const int bytes = fwd_layout(N, a.K, fused).total;
    if (a.nseg > 1) {
        e = launch_dyn(pdssm_fwd_kernel<N, true>, dim3(gx, a.B, a.nseg - 1), bytes, st, a);
        if (e != cudaSuccess) return e;
        const int64_t groups = (int64_t)a.B * a.H * N;
        pdssm_carry_fwd_kernel<N><<<(unsigned)((groups + NT - 1) / NT), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return launch_dyn(pdssm_fwd_kernel<N, false>, dim3(gx, a.B, a.nseg), bytes, st, a);
}

template <int N>
cudaError_t bwd_impl(const PdArgs& a, cudaStream_t st) {
    constexpr int SEQ = NT / N;
    const bool fused = SEQ * a.K <= SCORE_ROW_MAX;
    const unsigned gx = (unsigned)((a.H + SEQ - 1) / SEQ);
    cudaError_t e;
    if (a.nseg > 1) {
        pdssm_bwd_summary_kernel<N><<<dim3(gx, a.B, a.nseg - 1), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t groups = (int64_t)a.B * a.H * N;
        pdssm_carry_bwd_kernel<N><<<(unsigned)((groups + NT - 1) / NT), NT, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const unsigned gxb = (unsigned)((a.H + BW_PAIRS * (32 / N) - 1) / (BW_PAIRS * (32 / N)));
    e = launch_dyn(pdssm_bwd_kernel<N>, dim3(gxb, a.B, a.nseg), bwd_layout(N, a.K, fused).total, st, a);
    if (e != cudaSuccess || fused) return e;
    const int64_t n = (int64_t)a.B * a.L * a.H;
    pdssm_dscores_kernel<N><<<(unsigned)((n + NT - 1) / NT), NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Kernels one call launches: the forward's select (when not fused), segment summaries and carry,
// and scan; the backward's segment summaries and carry, scan, and score gradient (when not fused).
int pdssm_launches(const PdArgs& a) {
    const bool fused = (NT / a.N) * a.K <= SCORE_ROW_MAX;
    return (fused ? 0 : 1) + (a.nseg > 1 ? 2 : 0) + 1;
}

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
