// Step-size projection in front of the real scan ("选择性状态空间模型(S3M)原理与工程实践" §1.1:
// delta = softplus(projection(x)); §4.1 fuses the discretisation with this matrix product).  Per
// row m = (batch, step):  delta_raw[m, d] = sum_r u[m, r] w[d, r] + bias[d],  with backward
//   du = g w,   dw = g^T u,   dbias = sum_m g       (g = dL / d delta_raw).
// Three tensor-core GEMMs, bf16 operands and fp32 accumulation (mma.sync m16n8k16, operands
// staged through shared memory by cp.async and loaded into fragments with ldmatrix, transposed
// where the operand is stored the other way round):
//   forward   [M x D] = u [M x R] . w [D x R]^T, epilogue + bias, bf16 out;
//   du        [M x R] = g [M x D] . w [D x R];
//   dw, dbias [D x (R+1)] = g^T [D x M] . (u | 1) [M x (R+1)], split over M into fixed-order
//             partial sums (the ones column gives dbias), then a reduction.
// The rank R is small (tens to a few hundred), so each GEMM moves far more bytes than it does
// arithmetic per byte: they are bound by HBM (writing delta_raw, reading g), not by the tensor pipe.
#include <cuda_bf16.h>

#include "ssm_device.cuh"
#include "ssm_internal.h"

namespace ssm {
namespace {

constexpr int GT = 256;  // threads per CTA (8 warps)
constexpr int PAD = 8;   // bf16 padding per shared row (16 bytes: ldmatrix rows hit distinct banks)

__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp16(void* dst, const void* src, bool ok) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(ok ? 16 : 0));
}
__device__ __forceinline__ void ldsm4(unsigned (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p))
                 : "memory");
}
__device__ __forceinline__ void ldsm4t(unsigned (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p))
                 : "memory");
}
// D = A (16x16 bf16, row) . B (16x8 bf16, col) + C, fp32
__device__ __forceinline__ void mma16816(float (&c)[4], const unsigned (&a)[4], unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

enum Epi { EPI_BIAS_BF16 = 0, EPI_BF16 = 1, EPI_F32_PART = 2 };

struct GemmArgs {
    const __nv_bfloat16* A;  // logical [M][K]: AT ? A[k*lda + m] : A[m*lda + k]
    const __nv_bfloat16* B;  // logical [N][K]: BT ? B[k*ldb + n] : B[n*ldb + k]
    int64_t lda, ldb, ldc;
    int64_t M, N, K;         // N counts the ones column when ones_col >= 0
    int64_t kchunk;          // k range of one split (blockIdx.z)
    int ones_col;            // logical column of B that is all ones (dbias), or -1
    void* C;
    const float* bias;
};

// Shared-memory bytes of one configuration: a STAGES-deep ring of A and B tiles, reused for the
// bf16 output tile after the main loop.
template <bool AT, bool BT, int BM, int BN, int BK, int STAGES, int EPI>
struct GemmSmem {
    static constexpr int SA = AT ? BM + PAD : BK + PAD;  // shared row lengths (bf16)
    static constexpr int SB = BT ? BN + PAD : BK + PAD;
    static constexpr int A_ELEMS = AT ? BK * SA : BM * SA;
    static constexpr int B_ELEMS = BT ? BK * SB : BN * SB;
    static constexpr int SC = BN + PAD;  // bf16 output tile staged for 16-byte row stores
    static constexpr int PIPE_BYTES = STAGES * (A_ELEMS + B_ELEMS) * 2;
    static constexpr int C_BYTES = EPI == EPI_F32_PART ? 0 : BM * SC * 2;
    static constexpr int BYTES = PIPE_BYTES > C_BYTES ? PIPE_BYTES : C_BYTES;
};

// C tile [BM x BN] of blockIdx (y: m, x: n, z: k split).  Warps WM x WN, warp tile
// (BM/WM) x (BN/WN) of m16 x n8 mma tiles; k in steps of BK through a STAGES-deep cp.async ring.
template <bool AT, bool BT, int BM, int BN, int BK, int STAGES, int WM, int WN, int EPI>
__global__ void __launch_bounds__(GT) dtp_gemm_kernel(GemmArgs p) {
    static_assert(WM * WN * 32 == GT, "eight warps");
    static_assert(BK % 16 == 0 && STAGES >= 2, "k steps of whole mma blocks");
    constexpr int TM = BM / WM, TN = BN / WN, MT = TM / 16, NT8 = TN / 8;
    static_assert(TM % 16 == 0 && TN % 16 == 0, "warp tile of whole m16 x n16 blocks");
    using Sm = GemmSmem<AT, BT, BM, BN, BK, STAGES, EPI>;
    constexpr int SA = Sm::SA, SB = Sm::SB, A_ELEMS = Sm::A_ELEMS, B_ELEMS = Sm::B_ELEMS, SC = Sm::SC;
    extern __shared__ __align__(16) unsigned char smem[];
    __nv_bfloat16 (*sA)[A_ELEMS] = reinterpret_cast<__nv_bfloat16 (*)[A_ELEMS]>(smem);
    __nv_bfloat16 (*sB)[B_ELEMS] =
        reinterpret_cast<__nv_bfloat16 (*)[B_ELEMS]>(smem + STAGES * A_ELEMS * 2);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp / WN, wn = warp % WN;
    const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
    const int64_t kb = (int64_t)blockIdx.z * p.kchunk;
    const int64_t ke = min(p.K, kb + p.kchunk);
    const int nk = (int)((ke - kb + BK - 1) / BK);

    auto load = [&](int st, int64_t k0) {
        __nv_bfloat16* a = sA[st];
        __nv_bfloat16* b = sB[st];
        if (AT) {  // BK rows of k, BM/8 chunks of m
            for (int q = tid; q < BK * (BM / 8); q += GT) {
                const int r = q / (BM / 8), c = q % (BM / 8);
                const int64_t k = k0 + r, m = m0 + 8 * c;
                const bool ok = k < ke && m + 8 <= p.M;
                cp16(a + r * SA + 8 * c, ok ? p.A + k * p.lda + m : p.A, ok);
            }
        } else {   // BM rows of m, BK/8 chunks of k
            for (int q = tid; q < BM * (BK / 8); q += GT) {
                const int r = q / (BK / 8), c = q % (BK / 8);
                const int64_t m = m0 + r, k = k0 + 8 * c;
                const bool ok = m < p.M && k + 8 <= ke;
                cp16(a + r * SA + 8 * c, ok ? p.A + m * p.lda + k : p.A, ok);
            }
        }
        if (BT) {  // BK rows of k, BN/8 chunks of n; the ones column's chunk is written directly
            for (int q = tid; q < BK * (BN / 8); q += GT) {
                const int r = q / (BN / 8), c = q % (BN / 8);
                const int64_t k = k0 + r, n = n0 + 8 * c;
                __nv_bfloat16* dst = b + r * SB + 8 * c;
                if (p.ones_col >= 0 && n == p.ones_col) {
                    const __nv_bfloat16 one = __float2bfloat16(k < ke ? 1.0f : 0.0f);
                    const __nv_bfloat16 zero = __float2bfloat16(0.0f);
                    dst[0] = one;
#pragma unroll
                    for (int i = 1; i < 8; ++i) dst[i] = zero;
                } else {
                    const bool ok = k < ke && n + 8 <= (p.ones_col >= 0 ? p.ones_col : p.N);
                    cp16(dst, ok ? p.B + k * p.ldb + n : p.B, ok);
                }
            }
        } else {   // BN rows of n, BK/8 chunks of k
            for (int q = tid; q < BN * (BK / 8); q += GT) {
                const int r = q / (BK / 8), c = q % (BK / 8);
                const int64_t n = n0 + r, k = k0 + 8 * c;
                const bool ok = n < p.N && k + 8 <= ke;
                cp16(b + r * SB + 8 * c, ok ? p.B + n * p.ldb + k : p.B, ok);
            }
        }
        asm volatile("cp.async.commit_group;\n" ::);
    };

    const int g = lane >> 2, t4 = lane & 3;
    float bias_r[NT8][2];  // the bias of this thread's output columns, fetched before the main loop
#pragma unroll
    for (int jn = 0; jn < NT8; ++jn) {
        const int64_t col = n0 + wn * TN + 8 * jn + 2 * t4;
        const bool on = EPI == EPI_BIAS_BF16 && p.bias != nullptr && col < p.N;
        bias_r[jn][0] = on ? p.bias[col] : 0.0f;
        bias_r[jn][1] = on ? p.bias[col + 1] : 0.0f;
    }

    float acc[MT][NT8][4];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NT8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

    // ring: STAGES - 1 tiles in flight ahead of the one being multiplied (empty groups past the
    // end keep the group count uniform)
#pragma unroll
    for (int s0 = 0; s0 < STAGES - 1; ++s0) {
        if (s0 < nk)
            load(s0, kb + (int64_t)s0 * BK);
        else
            asm volatile("cp.async.commit_group;\n" ::);
    }
    for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % STAGES;
        asm volatile("cp.async.wait_group %0;\n" ::"n"(STAGES - 2));
        __syncthreads();  // tile kt is in; every thread is done with tile kt - 1
        {
            const int kn = kt + STAGES - 1;
            if (kn < nk)
                load(kn % STAGES, kb + (int64_t)kn * BK);
            else
                asm volatile("cp.async.commit_group;\n" ::);
        }
        const __nv_bfloat16* a = sA[st];
        const __nv_bfloat16* b = sB[st];
#pragma unroll
        for (int ks = 0; ks < BK / 16; ++ks) {
            unsigned af[MT][4];
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int mr = wm * TM + 16 * i;
                const int j = lane >> 3;
                if (AT)  // stored [k][m]: matrix j = (m block j&1, k block j>>1)
                    ldsm4t(af[i], a + (ks * 16 + 8 * (j >> 1) + (lane & 7)) * SA + mr + 8 * (j & 1));
                else     // stored [m][k]: lanes 0-15 rows m, lanes 16-31 the upper k half
                    ldsm4(af[i], a + (mr + (lane & 15)) * SA + ks * 16 + 8 * (lane >> 4));
            }
#pragma unroll
            for (int jn = 0; jn < NT8; jn += 2) {
                const int nc = wn * TN + 8 * jn;
                const int j = lane >> 3;
                unsigned bf[4];  // (b0b1, b2b3) of n8 tile jn, then of tile jn + 1
                if (BT)  // stored [k][n]: matrix j = (k block j&1, n block j>>1)
                    ldsm4t(bf, b + (ks * 16 + 8 * (j & 1) + (lane & 7)) * SB + nc + 8 * (j >> 1));
                else     // stored [n][k]: matrix j = (n block j>>1, k block j&1)
                    ldsm4(bf, b + (nc + 8 * (j >> 1) + (lane & 7)) * SB + ks * 16 + 8 * (j & 1));
#pragma unroll
                for (int i = 0; i < MT; ++i) {
                    mma16816(acc[i][jn], af[i], bf[0], bf[1]);
                    mma16816(acc[i][jn + 1], af[i], bf[2], bf[3]);
                }
            }
        }
    }
    __syncthreads();  // every thread is done with the ring (the output tile reuses it)

    // epilogue: c0, c1 at (row g, cols 2t, 2t+1), c2, c3 at row g + 8
    if (EPI == EPI_F32_PART) {
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int jn = 0; jn < NT8; ++jn) {
                const int64_t col = n0 + wn * TN + 8 * jn + 2 * t4;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t row = m0 + wm * TM + 16 * i + g + 8 * h;
                    if (row >= p.M || col >= p.N) continue;
                    float* c = static_cast<float*>(p.C) + (int64_t)blockIdx.z * p.M * p.ldc + row * p.ldc;
                    c[col] = acc[i][jn][2 * h];
                    if (col + 1 < p.N) c[col + 1] = acc[i][jn][2 * h + 1];
                }
            }
        return;
    }
    // bf16 outputs (N a multiple of 8): the tile goes through shared memory (the pipeline buffers
    // are free after the last barrier) and leaves as 16-byte row pieces
    __nv_bfloat16* sC = reinterpret_cast<__nv_bfloat16*>(smem);
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int jn = 0; jn < NT8; ++jn) {
            const int cl = wn * TN + 8 * jn + 2 * t4;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int rl = wm * TM + 16 * i + g + 8 * h;
                *reinterpret_cast<__nv_bfloat162*>(sC + rl * SC + cl) = __floats2bfloat162_rn(
                    acc[i][jn][2 * h] + bias_r[jn][0], acc[i][jn][2 * h + 1] + bias_r[jn][1]);
            }
        }
    __syncthreads();
    for (int q = tid; q < BM * (BN / 8); q += GT) {
        const int rl = q / (BN / 8), c8 = q % (BN / 8);
        const int64_t row = m0 + rl, col = n0 + 8 * c8;
        if (row < p.M && col < p.N)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + row * p.ldc + col) =
                *reinterpret_cast<const uint4*>(sC + rl * SC + 8 * c8);
    }
}

// dw[d, r] = sum_s part[s, d, r] (r < R), dbias[d] = sum_s part[s, d, R], in a fixed order.
__global__ void dtp_reduce_kernel(const float* __restrict__ part, int splits, int64_t D, int R,
                                  float* __restrict__ dw, float* __restrict__ dbias) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = D * (R + 1);
    if (i >= n) return;
    const int64_t d = i / (R + 1);
    const int r = (int)(i - d * (R + 1));
    // four interleaved running sums (independent loads in flight), combined in a fixed order
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    int k = 0;
    for (; k + 4 <= splits; k += 4) {
        s0 += part[(int64_t)k * n + i];
        s1 += part[(int64_t)(k + 1) * n + i];
        s2 += part[(int64_t)(k + 2) * n + i];
        s3 += part[(int64_t)(k + 3) * n + i];
    }
    for (; k < splits; ++k) s0 += part[(int64_t)k * n + i];
    const float s = (s0 + s1) + (s2 + s3);
    if (r < R)
        dw[d * R + r] = s;
    else if (dbias)
        dbias[d] = s;
}

template <bool AT, bool BT, int BM, int BN, int BK, int STAGES, int WM, int WN, int EPI>
cudaError_t run_gemm(const GemmArgs& a, int splits, cudaStream_t st) {
    const dim3 grid((unsigned)((a.N + BN - 1) / BN), (unsigned)((a.M + BM - 1) / BM), (unsigned)splits);
    constexpr int bytes = GemmSmem<AT, BT, BM, BN, BK, STAGES, EPI>::BYTES;
    auto kern = dtp_gemm_kernel<AT, BT, BM, BN, BK, STAGES, WM, WN, EPI>;
    if (bytes > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, GT, bytes, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int64_t dtproj_rows_per_split() { return 256; }

cudaError_t launch_dtproj_fwd(const DtArgs& d, cudaStream_t st) {
    GemmArgs a = {};
    a.A = static_cast<const __nv_bfloat16*>(d.u);
    a.B = static_cast<const __nv_bfloat16*>(d.w);
    a.lda = d.R; a.ldb = d.R; a.ldc = d.D;
    a.M = d.M; a.N = d.D; a.K = d.R; a.kchunk = d.R;
    a.ones_col = -1;
    a.C = d.delta_raw;
    a.bias = d.bias;
    // R <= 64: the whole k range in one shared tile (no ring turnover); larger R: 128-row tiles
    // so each w tile serves twice the rows
    if (d.R <= 16) return run_gemm<false, false, 64, 128, 16, 2, 2, 4, EPI_BIAS_BF16>(a, 1, st);
    if (d.R <= 32) return run_gemm<false, false, 64, 128, 32, 2, 2, 4, EPI_BIAS_BF16>(a, 1, st);
    if (d.R <= 48) return run_gemm<false, false, 64, 128, 48, 2, 2, 4, EPI_BIAS_BF16>(a, 1, st);
    if (d.R <= 64) return run_gemm<false, false, 64, 128, 64, 2, 2, 4, EPI_BIAS_BF16>(a, 1, st);
    return run_gemm<false, false, 128, 128, 64, 2, 2, 4, EPI_BIAS_BF16>(a, 1, st);
}

cudaError_t launch_dtproj_bwd(const DtArgs& d, cudaStream_t st) {
    // du [M x R] = g [M x D] . w [D x R]   (B stored [k = d][n = r])
    GemmArgs a = {};
    a.A = static_cast<const __nv_bfloat16*>(d.g);
    a.B = static_cast<const __nv_bfloat16*>(d.w);
    a.lda = d.D; a.ldb = d.R; a.ldc = d.R;
    a.M = d.M; a.N = d.R; a.K = d.D; a.kchunk = d.D;
    a.ones_col = -1;
    a.C = d.du;
    cudaError_t e = run_gemm<false, true, 128, 64, 64, 3, 4, 2, EPI_BF16>(a, 1, st);
    if (e != cudaSuccess) return e;
    // partials [split][D][R+1] = g^T [D x M] . (u | 1) [M x (R+1)]   (A stored [k = m][d], B [m][r])
    GemmArgs b = {};
    b.A = static_cast<const __nv_bfloat16*>(d.g);
    b.B = static_cast<const __nv_bfloat16*>(d.u);
    b.lda = d.D; b.ldb = d.R; b.ldc = d.R + 1;
    b.M = d.D; b.N = d.R + 1; b.K = d.M; b.kchunk = dtproj_rows_per_split();
    b.ones_col = d.R;
    b.C = d.part;
    e = run_gemm<true, true, 128, 64, 32, 3, 4, 2, EPI_F32_PART>(b, d.splits, st);
    if (e != cudaSuccess) return e;
    const int64_t n = d.D * (d.R + 1);
    dtp_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(d.part, d.splits, d.D, d.R, d.dw,
                                                                    d.dbias);
    return cudaGetLastError();
}

}  // namespace ssm
