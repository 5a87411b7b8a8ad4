// Step-size projection in front of the real scan ("选择性状态空间模型(S3M)原理与工程实践" §1.1:
// delta = softplus(projection(x)); §4.1 fuses the discretisation with this matrix product).  Per
// row m = (batch, step):  delta_raw[m, d] = sum_r u[m, r] w[d, r] + bias[d],  with backward
//   du = g w,   dw = g^T u,   dbias = sum_m g       (g = dL / d delta_raw).
// Three GEMMs on the fifth-generation tensor cores (tcgen05.mma, kind::f16: bf16 operands from
// shared memory, fp32 accumulator in tensor memory), all from one kernel template:
//   forward   C [M x D]   = u [M x R] . w [D x R]^T  (both operands k-major), + bias, bf16 out;
//   du        C [M x R]   = g [M x D] . w [D x R]    (w read n-major: its rows run along k);
//   dw, dbias C [D x R+1] = g^T [D x M] . (u | 1)    (both operands m/n-major; split over M into
//             fixed-order fp32 partial sums; a second MMA per step against a static shared block
//             whose first column is ones gives dbias), then a reduction.
// Operand tiles are 64 elements wide (one 128-byte swizzle atom of bf16) and reach shared memory by
// TMA (cp.async.bulk.tensor, 128-byte swizzle, out-of-range rows and columns filled with zeros) in
// the canonical layouts the tensor core reads through its shared-memory descriptors: k-major
// tiles as rows of 64 k-elements, m/n-major tiles as rows of 64 m/n-elements per k, so every box is
// a plain 2-D window of a global array.  One thread issues the copies and another the MMAs (four
// k16 steps per stage); mbarriers carry "stage full" (TMA transaction bytes) and "stage free" /
// "accumulator ready" (tcgen05.commit); the forward also has drain warps of its own (see
// dtp_fwd_ws_kernel).  The issue / wait order and the phase parities are model-checked on the host
// by tests/test_mbarrier_protocol.py.
// The rank R is small (tens to a few hundred), so each GEMM moves far more bytes than it does
// arithmetic per byte: they are bound by HBM (writing delta_raw, reading g), not by the tensor pipe.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ssm_device.cuh"
#include "ssm_internal.h"

namespace ssm {
namespace {

constexpr int TM = 128;    // UMMA M: tile rows = tensor-memory lanes
constexpr int BK = 64;     // k depth of one stage: one 128-byte swizzle atom of bf16
constexpr int NTH = 128;   // 4 warps: loaders and epilogue; thread 0 also issues the MMAs
constexpr int A_BYTES = TM * 128;          // one A stage (either layout)
constexpr unsigned kSpinLimit = 1u << 20;  // bounded mbarrier waits (well above any MMA)

__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void st_shared_v4(unsigned a, unsigned x, unsigned y, unsigned z, unsigned w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
// generic-proxy writes of this thread (plain shared stores) become visible to the tensor core's
// reads through the async proxy
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_init(unsigned a, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned a, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}
// arrival that also announces `bytes` of TMA transactions still to land on this phase
__device__ __forceinline__ void mbar_expect_tx(unsigned a, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(a), "r"(bytes) : "memory");
}
// 2-D tensor-map box at (x innermost, y) into shared memory, completing on mbarrier `bar`
__device__ __forceinline__ void tma_load_2d(unsigned dst, const CUtensorMap* map, int x, int y, unsigned bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// 2-D tensor-map box from shared memory to (x innermost, y); rows and columns outside the array
// are not written
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, unsigned src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// this thread's bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
// true once the phase of parity `parity` has completed; false if the bounded wait gave up.  The
// caller must not be two or more phases behind (parity alone cannot tell those apart).
__device__ __forceinline__ bool mbar_wait(unsigned a, unsigned parity) {
    for (unsigned i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(a, parity)) return true;
    return false;
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// D[tmem] (+)= A[smem] . B[smem]^T, one kind::f16 instruction (M = 128, N, K = 16)
__device__ __forceinline__ void umma_bf16(unsigned d, uint64_t adesc, uint64_t bdesc, unsigned idesc,
                                          unsigned accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
// arrive on the mbarrier once every MMA this thread issued so far has completed
__device__ __forceinline__ void umma_commit(unsigned mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar)
                 : "memory");
}
// 32 consecutive fp32 accumulator columns of this warp's 32 tensor-memory lanes (one row per lane)
__device__ __forceinline__ void tmem_ld32(unsigned taddr, float (&v)[32]) {
    unsigned r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start, leading and stride
// byte offsets in 16-byte units at bits 0, 16, 32; version 1 at bit 46; layout 2 at bit 61).
__device__ __forceinline__ uint64_t sw128_desc(unsigned saddr, unsigned lbo, unsigned sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, operand majors, N, M = 128.
__host__ __device__ constexpr unsigned idesc_bf16(int n, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((unsigned)a_mn << 15) | ((unsigned)b_mn << 16) |
           ((unsigned)(n >> 3) << 17) | ((unsigned)(TM >> 4) << 24);
}

// k-loop kernel epilogues: bf16 rows of C, or fp32 partial sums of one split
enum Epi { EPI_BF16 = 1, EPI_F32_PART = 2 };

struct TcArgs {
    int64_t M, N, K;         // logical C [M][N] = sum_k A(m, k) B(n, k); N counts the column sums
    int64_t ldc;             // bf16 outputs: row stride of C
    int64_t kchunk;          // k range of one split (blockIdx.z), a multiple of 64
    int64_t ones_out;        // EPI_F32_PART: data columns below it; the column sums (dbias) go to it
    void* C;                 // EPI_F32_PART: [split][N][M] fp32; else [M][N] bf16
    const float* bias;
    unsigned* status;        // workspace status word: SSM_ERR_TIMEOUT when a bounded wait gives up
};

__host__ __device__ constexpr int tmem_cols(int bn) {
    return bn <= 32 ? 32 : bn <= 64 ? 64 : bn <= 128 ? 128 : bn <= 256 ? 256 : 512;
}

// Shared layout of the k-loop kernel: STAGES x (A tile, B tile), the static block of ones (when
// the column sums are wanted), then the mbarriers.
template <int BN, int STAGES, bool ONES>
struct TcSmem {
    static constexpr int B_BYTES = BN * 128;                 // one B stage (either layout)
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int PIPE = STAGES * STAGE;
    static constexpr int ONE_BLK = PIPE;                     // 64 k rows x 64 columns, column 0 = 1
    static constexpr int FULL = ONE_BLK + (ONES ? BK * 128 : 0);  // STAGES "stage loaded"
    static constexpr int FREE = FULL + STAGES * 8;           // STAGES "stage consumed"
    static constexpr int DONE = FREE + STAGES * 8;           // all MMAs done
    static constexpr int SLOT = DONE + 8;                    // tensor-memory address
    static constexpr int BYTES = SLOT + 8 + 1024;            // + slack to align the base to 1024
    static constexpr int SROW = BN * 2 + 16;                 // bf16 output row staged for stores
    static_assert(TM * SROW <= PIPE, "output staging fits the pipeline buffers");
};

__device__ __forceinline__ void tmem_alloc_cta(unsigned slot, unsigned cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(slot), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_cta(unsigned taddr, unsigned cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(cols) : "memory");
}

// C tile [128 x BN] at tile coordinates (bn: n, bm: m, bz: k split), the k range in 64-deep
// stages.  mA, mB: tensor maps of A and B with 64-element-wide boxes (k-major: {64 k, rows};
// m/n-major: {64 m/n, 64 k}); they are kernel parameters (__grid_constant__), passed on by
// reference so the copies read them in parameter space.  ONES: one more 64-wide accumulator block
// multiplies A by a static block whose first column is all ones, giving A's column sums (dbias) in
// accumulator column BN.  The dynamic shared memory holds at least TcSmem<BN, STAGES, ONES>::BYTES.
template <bool A_MN, bool B_MN, int BN, int STAGES, bool ONES, int EPI>
__device__ __forceinline__ void tc_tile(const CUtensorMap& mA, const CUtensorMap& mB, const TcArgs& p,
                                        int bn, int bm, int bz, unsigned char* smem_raw) {
    static_assert(BN % 64 == 0 && BN <= 256 && STAGES >= 2, "n tile of whole 64-wide blocks");
    static_assert(!ONES || EPI == EPI_F32_PART, "column sums go to the fp32 partial sums");
    using Sm = TcSmem<BN, STAGES, ONES>;
    constexpr int TCOLS = tmem_cols(BN + (ONES ? 64 : 0));
    const unsigned raw = smem_u32(smem_raw);
    const unsigned base = (raw + 1023u) & ~1023u;   // swizzle atoms need 1024-byte alignment
    unsigned char* gbase = smem_raw + (base - raw);
    const unsigned full = base + Sm::FULL, free_ = base + Sm::FREE, done = base + Sm::DONE;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = (int64_t)bm * TM, n0 = (int64_t)bn * BN;
    const int64_t kb = (int64_t)bz * p.kchunk;
    const int64_t ke = min(p.K, kb + p.kchunk);
    const int nk = ke > kb ? (int)((ke - kb + BK - 1) / BK) : 0;

    if (warp == 0) tmem_alloc_cta(base + Sm::SLOT, TCOLS);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + 8 * s, 1);
            mbar_init(free_ + 8 * s, 1);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (ONES) {
        // 64 k rows x 64 columns (m/n-major, 128-byte swizzle), bf16 1.0 in column 0 of every row:
        // chunk 0 of row r sits at chunk (0 ^ (r & 7)).  Rows past K meet zeros in A.
        for (int q = tid; q < BK * 8; q += NTH) {
            const int r = q >> 3, c = q & 7;
            st_shared_v4(base + Sm::ONE_BLK + r * 128 + ((c ^ (r & 7)) << 4), c == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
        }
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tmem = *reinterpret_cast<volatile unsigned*>(gbase + Sm::SLOT);

    bool ok = true;
    auto issue = [&](int t, int st) {
        const unsigned a = base + st * Sm::STAGE, b = a + A_BYTES, f = full + 8 * st;
        const int k0 = (int)(kb + (int64_t)t * BK);
        mbar_expect_tx(f, Sm::STAGE);
        if (!A_MN) {
            tma_load_2d(a, &mA, k0, (int)m0, f);
        } else {
            tma_load_2d(a, &mA, (int)m0, k0, f);
            tma_load_2d(a + BK * 128, &mA, (int)m0 + 64, k0, f);
        }
        if (!B_MN) {
            tma_load_2d(b, &mB, k0, (int)n0, f);
        } else {
#pragma unroll
            for (int blk = 0; blk < BN / 64; ++blk) tma_load_2d(b + blk * (BK * 128), &mB, (int)n0 + 64 * blk, k0, f);
        }
    };
    if (tid == 0) {
        // copies: tile t into stage t % STAGES once the MMAs of tile t - STAGES have read it
        for (int t = 0; t < nk; ++t) {
            const int st = t % STAGES;
            if (t >= STAGES && !(ok = mbar_wait(free_ + 8 * st, (unsigned)((t / STAGES - 1) & 1)))) break;
            issue(t, st);
        }
    } else if (tid == 32) {
        // MMAs, one stage at a time as its copies land
        for (int kt = 0; kt < nk; ++kt) {
            const int s = kt % STAGES;
            if (!(ok = mbar_wait(full + 8 * s, (unsigned)((kt / STAGES) & 1)))) break;
            const unsigned a = base + s * Sm::STAGE, b = a + A_BYTES;
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < BK / 16; ++j) {
                // k16 step j: 32 bytes into each k-major row, or two 8-row groups of k rows
                const uint64_t ad = A_MN ? sw128_desc(a + j * 2048, BK * 128, 1024)
                                         : sw128_desc(a + j * 32, 16, 1024);
                const uint64_t bd = B_MN ? sw128_desc(b + j * 2048, BK * 128, 1024)
                                         : sw128_desc(b + j * 32, 16, 1024);
                umma_bf16(tmem, ad, bd, idesc_bf16(BN, A_MN, B_MN), (kt | j) != 0);
                if (ONES)
                    umma_bf16(tmem + BN, ad, sw128_desc(base + Sm::ONE_BLK + j * 2048, BK * 128, 1024),
                              idesc_bf16(64, A_MN, true), (kt | j) != 0);
            }
            umma_commit(free_ + 8 * s);
        }
        umma_commit(done);  // arrives once every MMA issued above has completed
        if (ok) ok = mbar_wait(done, 0);
        tc_fence_before();
    }
    // the other threads wait here (not spinning on the mbarriers beside threads 0 and 32)
    const bool bad = __syncthreads_or(!ok);
    tc_fence_after();

    if (!bad) {
        const int row = warp * 32 + lane;  // tile row = tensor-memory lane
        const unsigned tl = tmem + ((unsigned)(warp * 32) << 16);
        if (EPI == EPI_F32_PART) {
            // partial sums [split][N][M]: one column per store, the warp's 32 rows contiguous; tile
            // columns below ones_out are data columns, accumulator column BN the column sums
            float* out = static_cast<float*>(p.C) + (int64_t)bz * p.N * p.M;
            const int64_t m = m0 + row;
#pragma unroll 1
            for (int c0 = 0; c0 < BN + (ONES ? 32 : 0); c0 += 32) {
                float v[32];
                if (nk > 0) {
                    tmem_ld32(tl + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                }
                if (m < p.M) {
                    if (c0 < BN) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int64_t col = n0 + c0 + i;
                            if (col < p.ones_out) out[col * p.M + m] = v[i];
                        }
                    } else {
                        out[(int64_t)p.ones_out * p.M + m] = v[0];
                    }
                }
            }
        } else {
            // bf16 rows staged in shared memory (the pipeline buffers are free), then stored as
            // 16-byte row pieces
            const unsigned srow = base + row * Sm::SROW;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                float v[32];
                if (nk > 0) {
                    tmem_ld32(tl + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    unsigned w4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * q + 2 * i], v[8 * q + 2 * i + 1]);
                        w4[i] = *reinterpret_cast<const unsigned*>(&h);
                    }
                    st_shared_v4(srow + (c0 + 8 * q) * 2, w4[0], w4[1], w4[2], w4[3]);
                }
            }
            __syncthreads();
            for (int q = tid; q < TM * (BN / 8); q += NTH) {
                const int rl = q / (BN / 8), c8 = q % (BN / 8);
                const int64_t m = m0 + rl, col = n0 + 8 * c8;
                if (m < p.M && col < p.N)
                    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + m * p.ldc + col) =
                        *reinterpret_cast<const uint4*>(gbase + rl * Sm::SROW + 16 * c8);
            }
        }
    } else {
        if (tid == 0) flag_status(p.status, kStatusTimeout);
        if (tid == 32) mbar_wait(done, 0);  // the MMAs already issued get a last bounded chance
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_cta(tmem, TCOLS);
    }
}

// One GEMM: tile (blockIdx.x: n, blockIdx.y: m, blockIdx.z: k split)
template <bool A_MN, bool B_MN, int BN, int STAGES, bool ONES, int EPI>
__global__ void __launch_bounds__(NTH) dtp_tc_kernel(const __grid_constant__ CUtensorMap mA,
                                                     const __grid_constant__ CUtensorMap mB, TcArgs p) {
    extern __shared__ unsigned char smem_raw[];
    tc_tile<A_MN, B_MN, BN, STAGES, ONES, EPI>(mA, mB, p, blockIdx.x, blockIdx.y, blockIdx.z, smem_raw);
}

// The projection's two backward GEMMs in one launch, so that both stream g at once: CTAs
// [0, n_du) compute du (one 128-row tile of g each, the whole k = D range), the others one
// (d tile, row split) of the dw / dbias partial sums.  For R <= 64.
constexpr int BWD_DU_STAGES = 4, BWD_DW_STAGES = 4;
__global__ void __launch_bounds__(NTH) dtp_bwd_kernel(const __grid_constant__ CUtensorMap gK,
                                                      const __grid_constant__ CUtensorMap wN,
                                                      const __grid_constant__ CUtensorMap gM,
                                                      const __grid_constant__ CUtensorMap uN, TcArgs du,
                                                      TcArgs dw, int n_du, int dw_mt) {
    extern __shared__ unsigned char smem_raw[];
    const int c = blockIdx.x;
    if (c < n_du) {
        tc_tile<false, true, 64, BWD_DU_STAGES, false, EPI_BF16>(gK, wN, du, 0, c, 0, smem_raw);
    } else {
        const int j = c - n_du;
        tc_tile<true, true, 64, BWD_DW_STAGES, true, EPI_F32_PART>(gM, uN, dw, 0, j % dw_mt, j / dw_mt,
                                                                   smem_raw);
    }
}

// Forward GEMM, warp-specialised and persistent.  Work unit = one 128-row tile of u times a run of
// up to NCH consecutive 64-row tiles of w (one output tile each); CTA c takes units c, c + G, ...
//   warp 0, one thread: TMA copies: the unit's u tile into one of two A buffers (once per unit),
//                       each w tile into a ring of STAGES stages;
//   warp 1, one thread: each output tile's MMAs into one of ACC tensor-memory accumulators (the
//                       warp also allocates and frees the tensor memory);
//   warps 2-5: drain.  Warp w reads accumulator lanes 32 (w % 4) .. + 31 (the quarter a warp may
//              reach), adds the bias, packs bf16 into its own 128-byte-swizzled staging box of
//              32 rows x 64 columns (two, alternating) and stores it with one TMA copy.
// No CTA-wide barrier inside the loop: "full" (TMA transaction bytes), "free" and "accumulator
// full" (tcgen05.commit) and "accumulator free" (one arrival per drain warp) mbarriers hand the
// tiles on, so copies, MMAs and drains of different tiles overlap.  Copying u once per unit rather
// than once per output tile matters: u's rows are R bf16 (96 bytes at R = 48), short, unaligned
// rows that the copy engine moves at a fraction of its rate for long ones.
constexpr int WS_NTH = 192;
constexpr int WS_BN = 64;
template <int KA, int STAGES, int ACC>
struct WsSm {
    static constexpr int A_ST = KA * TM * 128;          // u tile: KA swizzle atoms of 128 rows
    static constexpr int B_ST = KA * WS_BN * 128;       // w tile: KA atoms of 64 rows
    static constexpr int BST = 2 * A_ST;                // the ring of w stages after two A buffers
    static constexpr int BOX = 32 * 128;                // staging box: 32 rows x 64 bf16
    static constexpr int EPI = BST + STAGES * B_ST;     // 4 warps x 2 boxes
    // afull, afree [2]; full, free [STAGES]; accf, acce [ACC]; done
    static constexpr int BAR = EPI + 4 * 2 * BOX;
    static constexpr int SLOT = BAR + (4 + 2 * STAGES + 2 * ACC + 1) * 8;
    static constexpr int BYTES = SLOT + 8 + 1024;       // + slack to align the base to 1024
};

__device__ __forceinline__ void mbar_arrive(unsigned a) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(a) : "memory");
}
// this thread's bulk stores but the most recent one have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() {
    asm volatile("cp.async.bulk.wait_group.read 1;\n" ::: "memory");
}

template <int KA, int STAGES, int ACC>
__global__ void __launch_bounds__(WS_NTH, 1) dtp_fwd_ws_kernel(const __grid_constant__ CUtensorMap mA,
                                                               const __grid_constant__ CUtensorMap mB,
                                                               const __grid_constant__ CUtensorMap mC,
                                                               TcArgs p, int n_nt, int nch, int64_t nunits) {
    using Sm = WsSm<KA, STAGES, ACC>;
    constexpr int BN = WS_BN;
    constexpr int TCOLS = tmem_cols(ACC * BN);
    static_assert(ACC * BN <= 512 && STAGES >= 2, "accumulators fit tensor memory");
    extern __shared__ unsigned char smem_raw[];
    const unsigned raw = smem_u32(smem_raw);
    const unsigned base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const unsigned bar = base + Sm::BAR;
    auto afull = [&](int k) { return bar + 8 * k; };
    auto afree = [&](int k) { return bar + 8 * (2 + k); };
    auto full = [&](int s) { return bar + 8 * (4 + s); };
    auto freeb = [&](int s) { return bar + 8 * (4 + STAGES + s); };
    auto accf = [&](int a) { return bar + 8 * (4 + 2 * STAGES + a); };
    auto acce = [&](int a) { return bar + 8 * (4 + 2 * STAGES + ACC + a); };
    const unsigned done = bar + 8 * (4 + 2 * STAGES + 2 * ACC);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nchk = (n_nt + nch - 1) / nch;  // n runs per 128-row tile of u
    // unit k of this CTA: 128-row tile of u and first n tile, number of n tiles
    auto unit = [&](int64_t k, int64_t& m0, int& nt0, int& nj) {
        const int64_t g = (int64_t)blockIdx.x + k * gridDim.x;
        m0 = g / nchk * TM;
        nt0 = (int)(g % nchk) * nch;
        nj = n_nt - nt0 < nch ? n_nt - nt0 : nch;
    };
    const int64_t U = (int64_t)blockIdx.x < nunits ? (nunits - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (warp == 1) tmem_alloc_cta(base + Sm::SLOT, TCOLS);
    if (tid == 0) {
        for (int k = 0; k < 2; ++k) {
            mbar_init(afull(k), 1);
            mbar_init(afree(k), 1);
        }
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(freeb(s), 1);
        }
        for (int a = 0; a < ACC; ++a) {
            mbar_init(accf(a), 1);
            mbar_init(acce(a), 4);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tmem = *reinterpret_cast<volatile unsigned*>(gbase + Sm::SLOT);

    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            int i = 0;  // output tiles so far
            for (int64_t k = 0; k < U && ok; ++k) {
                int64_t m0;
                int nt0, nj;
                unit(k, m0, nt0, nj);
                const int ab = (int)(k & 1);
                // the A buffer last held unit k - 2: its MMAs must be done
                if (k >= 2 && !(ok = mbar_wait(afree(ab), (unsigned)(((k >> 1) - 1) & 1)))) break;
                const unsigned a = base + ab * Sm::A_ST;
                mbar_expect_tx(afull(ab), Sm::A_ST);
#pragma unroll
                for (int at = 0; at < KA; ++at) tma_load_2d(a + at * (TM * 128), &mA, 64 * at, (int)m0, afull(ab));
                for (int j = 0; j < nj; ++j, ++i) {
                    const int s = i % STAGES, r = i / STAGES;
                    // the stage last held tile i - STAGES: its MMAs must be done
                    if (r >= 1 && !(ok = mbar_wait(freeb(s), (unsigned)((r - 1) & 1)))) break;
                    const unsigned b = base + Sm::BST + s * Sm::B_ST;
                    mbar_expect_tx(full(s), Sm::B_ST);
#pragma unroll
                    for (int at = 0; at < KA; ++at)
                        tma_load_2d(b + at * (BN * 128), &mB, 64 * at, (nt0 + j) * BN, full(s));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int i = 0;
            for (int64_t k = 0; k < U && ok; ++k) {
                int64_t m0;
                int nt0, nj;
                unit(k, m0, nt0, nj);
                const int ab = (int)(k & 1);
                if (!(ok = mbar_wait(afull(ab), (unsigned)((k >> 1) & 1)))) break;
                const unsigned a = base + ab * Sm::A_ST;
                for (int j = 0; j < nj; ++j, ++i) {
                    const int s = i % STAGES, ac = i % ACC;
                    if (!(ok = mbar_wait(full(s), (unsigned)((i / STAGES) & 1)))) break;
                    // the accumulator last held tile i - ACC: all four drain warps must have read it
                    if (i >= ACC && !(ok = mbar_wait(acce(ac), (unsigned)((i / ACC - 1) & 1)))) break;
                    tc_fence_after();
                    const unsigned b = base + Sm::BST + s * Sm::B_ST;
#pragma unroll
                    for (int jj = 0; jj < 4 * KA; ++jj)
                        umma_bf16(tmem + ac * BN,
                                  sw128_desc(a + (jj >> 2) * (TM * 128) + (jj & 3) * 32, 16, 1024),
                                  sw128_desc(b + (jj >> 2) * (BN * 128) + (jj & 3) * 32, 16, 1024),
                                  idesc_bf16(BN, false, false), jj != 0);
                    umma_commit(freeb(s));
                    umma_commit(accf(ac));
                }
                umma_commit(afree(ab));  // once the unit's MMAs are done, its A buffer is free
            }
            umma_commit(done);  // arrives once every MMA issued above has completed
        }
    } else {
        const int q = warp & 3;                               // accumulator lane quarter
        const unsigned tq = tmem + ((unsigned)(q * 32) << 16);
        const unsigned box0 = base + Sm::EPI + (warp - 2) * 2 * Sm::BOX;
        const bool has_bias = p.bias != nullptr;
        // bias of the tile's columns n0 + 2 lane and + 1 (lane pairs; a drain takes the other
        // lanes' pairs by shuffles), loaded one tile ahead so that its latency stays off the drain
        auto bias_pair = [&](int64_t n0) {
            const int64_t c = n0 + 2 * lane;  // N is a multiple of 8: c < N gives c + 1 < N
            return has_bias && c < p.N ? __ldg(reinterpret_cast<const float2*>(p.bias + c))
                                       : make_float2(0.0f, 0.0f);
        };
        int64_t m0n = 0;
        int nt0n = 0, njn = 0;
        if (U > 0) unit(0, m0n, nt0n, njn);
        float2 bnext = bias_pair((int64_t)nt0n * BN);
        int i = 0;
        for (int64_t k = 0; k < U && ok; ++k) {
            int64_t m0;
            int nt0, nj;
            unit(k, m0, nt0, nj);
            for (int j = 0; j < nj; ++j, ++i) {
                const int ac = i % ACC;
                const float2 bcur = bnext;
                // the next tile's bias: the next run of this unit, or the next unit's first
                if (j + 1 < nj) {
                    bnext = bias_pair((int64_t)(nt0 + j + 1) * BN);
                } else if (k + 1 < U) {
                    unit(k + 1, m0n, nt0n, njn);
                    bnext = bias_pair((int64_t)nt0n * BN);
                }
                if (!(ok = mbar_wait(accf(ac), (unsigned)((i / ACC) & 1)))) break;
                tc_fence_after();
                const int64_t n0 = (int64_t)(nt0 + j) * BN;
                const unsigned box = box0 + (i & 1) * Sm::BOX;
                if (lane == 0) bulk_wait_read_1();  // the store of tile i - 2 has read this box
                __syncwarp();
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    float v[32];
                    tmem_ld32(tq + ac * BN + c0, v);
                    if (has_bias) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            v[e] += __shfl_sync(0xffffffffu, bcur.x, (c0 + e) >> 1);
                            v[e + 1] += __shfl_sync(0xffffffffu, bcur.y, (c0 + e) >> 1);
                        }
                    }
                    // columns c0 .. c0 + 31: 16-byte chunks c0 / 8 + e of the box row `lane`, swizzled
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        unsigned w4[4];
#pragma unroll
                        for (int f = 0; f < 4; ++f) {
                            const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * e + 2 * f], v[8 * e + 2 * f + 1]);
                            w4[f] = *reinterpret_cast<const unsigned*>(&h);
                        }
                        const int cc = c0 / 8 + e;
                        st_shared_v4(box + lane * 128 + ((cc ^ (lane & 7)) << 4), w4[0], w4[1], w4[2], w4[3]);
                    }
                }
                tc_fence_before();
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(acce(ac));  // this warp's lanes of the accumulator are read
                    tma_store_2d(&mC, box, (int)n0, (int)m0 + q * 32);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }
    if (__syncthreads_or(!ok) && tid == 0) flag_status(p.status, kStatusTimeout);
    // every MMA issued has completed (bounded wait) before the tensor memory is freed
    if (warp == 1 && lane == 0) mbar_wait(done, 0);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_cta(tmem, TCOLS);
    }
}

// dw[d, r] = sum_s part[s, r, d] (r < R), dbias[d] = sum_s part[s, R, d], in a fixed order.
__global__ void dtp_reduce_kernel(const float* __restrict__ part, int splits, int64_t D, int R,
                                  float* __restrict__ dw, float* __restrict__ dbias) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // r * D + d
    const int64_t n = D * (R + 1);
    if (i >= n) return;
    const int r = (int)(i / D);
    const int64_t d = i - (int64_t)r * D;
    // splits in groups of 16 loads issued before any is used, summed in split order
    float s = 0.0f;
    for (int k0 = 0; k0 < splits; k0 += 16) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = k0 + k < splits ? __ldcs(part + (int64_t)(k0 + k) * n + i) : 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s += v[k];
    }
    if (r < R)
        dw[d * R + r] = s;
    else if (dbias)
        dbias[d] = s;
}

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point (no link to libcuda);
// looked up once (thread-safe initialisation of the function-local static)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        return nullptr;
    }();
    return fn;
}

// Tensor map of a row-major bf16 array [rows][cols] (row stride ld elements) with boxes of
// 64 columns x box_rows rows, 128-byte swizzle, zeros outside the array.
cudaError_t make_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <bool A_MN, bool B_MN, int BN, int STAGES, bool ONES, int EPI>
cudaError_t run_tc(const CUtensorMap& mA, const CUtensorMap& mB, const TcArgs& a, int splits, cudaStream_t st) {
    const int64_t ncols = ONES ? a.ones_out : a.N;  // data columns (the column sums ride along)
    const dim3 grid((unsigned)((ncols + BN - 1) / BN), (unsigned)((a.M + TM - 1) / TM), (unsigned)splits);
    constexpr int bytes = TcSmem<BN, STAGES, ONES>::BYTES;
    auto kern = dtp_tc_kernel<A_MN, B_MN, BN, STAGES, ONES, EPI>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, NTH, bytes, st>>>(mA, mB, a);
    return cudaGetLastError();
}

template <int KA, int STAGES, int ACC>
cudaError_t run_fwd(const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mC, const TcArgs& a,
                    cudaStream_t st) {
    constexpr int bytes = WsSm<KA, STAGES, ACC>::BYTES;
    auto kern = dtp_fwd_ws_kernel<KA, STAGES, ACC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100)) != cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // CTAs per SM: shared memory (with the per-CTA reservation) and the accumulators in the SM's
    // 512 tensor-memory columns bound it
    int smem_sm = 0, resv = 0;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&resv, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
    int per_sm = smem_sm / (bytes + resv);
    const int tcap = 512 / tmem_cols(ACC * WS_BN);
    if (per_sm > tcap) per_sm = tcap;
    if (per_sm < 1) per_sm = 1;
    const int64_t slots = (int64_t)sms * per_sm;
    const int n_nt = (int)((a.N + WS_BN - 1) / WS_BN);
    const int64_t n_mt = (a.M + TM - 1) / TM;
    // n tiles per unit: the run length that puts the fewest output tiles (plus one u copy per
    // unit, weighted as half a tile) on the busiest CTA
    int nch = n_nt;
    double best = -1.0;
    for (int k = 1; k <= n_nt && k <= 64; ++k) {  // k runs per u tile
        const int c = (n_nt + k - 1) / k;
        const int64_t units = n_mt * ((n_nt + c - 1) / c);
        const int64_t per = (units + slots - 1) / slots;
        const double cost = (double)per * c + 0.5 * (double)per;
        if (best < 0.0 || cost < best) {
            best = cost;
            nch = c;
        }
    }
    const int64_t nunits = n_mt * ((n_nt + nch - 1) / nch);
    const int64_t grid = nunits < slots ? nunits : slots;
    kern<<<(unsigned)grid, WS_NTH, bytes, st>>>(mA, mB, mC, a, n_nt, nch, nunits);
    return cudaGetLastError();
}

}  // namespace

// Rows of one dw / dbias split (a multiple of the 64-row stage)
// Rows of one dw / dbias split (a multiple of the 64-row stage).  R <= 64 runs du and dw in one
// launch: 1536-row splits give a dw CTA about the bytes of g of a du CTA, and both kinds fit one
// wave at two CTAs per SM for the workloads' row counts.
int64_t dtproj_rows_per_split(int R) { return R <= 64 ? 1536 : 1024; }

cudaError_t launch_dtproj_fwd(const DtArgs& d, cudaStream_t st) {
    // delta_raw [M x D] = u [M x R] . w [D x R]^T + bias: both operands k-major
    const int ka = (d.R + 63) / 64;              // 64-deep k atoms covering R, all in one stage
    CUtensorMap mA, mB, mC;
    cudaError_t e = make_map(&mA, d.u, d.M, d.R, d.R, TM);
    if (e == cudaSuccess) e = make_map(&mB, d.w, d.D, d.R, d.R, WS_BN);
    if (e == cudaSuccess) e = make_map(&mC, d.delta_raw, d.M, d.D, d.D, 32);  // a drain warp's box
    if (e != cudaSuccess) return e;
    TcArgs a = {};
    a.M = d.M; a.N = d.D; a.K = d.R; a.ldc = d.D; a.kchunk = d.R;
    a.ones_out = d.D;
    a.C = d.delta_raw;
    a.bias = d.bias;
    a.status = d.status;
    // w stages: four for one or two k atoms (two CTAs per SM for one), three and two beyond (one
    // CTA per SM)
    switch (ka) {
        case 1: return run_fwd<1, 4, 4>(mA, mB, mC, a, st);
        case 2: return run_fwd<2, 4, 4>(mA, mB, mC, a, st);
        case 3: return run_fwd<3, 3, 4>(mA, mB, mC, a, st);
        default: return run_fwd<4, 2, 4>(mA, mB, mC, a, st);
    }
}

cudaError_t launch_dtproj_bwd(const DtArgs& d, cudaStream_t st) {
    // du [M x R] = g [M x D] . w [D x R]: A = g k-major ({64 d, 128 rows} boxes), B = w read with its
    // rows along k (n-major, {64 r, 64 d} boxes)
    CUtensorMap gK, wN, gM, uN;
    cudaError_t e = make_map(&gK, d.g, d.M, d.D, d.D, TM);
    if (e == cudaSuccess) e = make_map(&wN, d.w, d.D, d.R, d.R, BK);
    // dw partials [split][R+1][D] = g^T [D x M] . (u | 1) [M x (R+1)]: A = g m-major and B = u
    // n-major ({64 d or r, 64 rows} boxes)
    if (e == cudaSuccess) e = make_map(&gM, d.g, d.M, d.D, d.D, BK);
    if (e == cudaSuccess) e = make_map(&uN, d.u, d.M, d.R, d.R, BK);
    if (e != cudaSuccess) return e;
    TcArgs a = {};
    a.M = d.M; a.N = d.R; a.K = d.D; a.ldc = d.R; a.kchunk = d.D;
    a.ones_out = d.R;
    a.C = d.du;
    a.status = d.status;
    // dw partials [split][R+1][D]: data columns 0..R-1, then the column sums of g (dbias) from the
    // static block of ones
    TcArgs b = {};
    b.M = d.D; b.N = d.R + 1; b.K = d.M; b.ldc = 0; b.kchunk = dtproj_rows_per_split(d.R);
    b.ones_out = d.R;
    b.C = d.part;
    b.status = d.status;
    const int64_t n = d.D * (d.R + 1);
    if (d.R <= 64) {
        // du and dw side by side in one launch
        constexpr int b_du = TcSmem<64, BWD_DU_STAGES, false>::BYTES;
        constexpr int b_dw = TcSmem<64, BWD_DW_STAGES, true>::BYTES;
        constexpr int bytes = b_du > b_dw ? b_du : b_dw;
        if ((e = cudaFuncSetAttribute(dtp_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
            cudaSuccess)
            return e;
        const int n_du = (int)((d.M + TM - 1) / TM);
        const int dw_mt = (int)((d.D + TM - 1) / TM);
        const int64_t ctas = (int64_t)n_du + (int64_t)dw_mt * d.splits;
        if (ctas > 0x7fffffff) return cudaErrorInvalidConfiguration;
        dtp_bwd_kernel<<<(unsigned)ctas, NTH, bytes, st>>>(gK, wN, gM, uN, a, b, n_du, dw_mt);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        dtp_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(d.part, d.splits, d.D, d.R, d.dw,
                                                                        d.dbias);
        return cudaGetLastError();
    }
    switch ((d.R + 63) / 64) {  // 64-wide n blocks covering R
        case 2: e = run_tc<false, true, 128, 6, false, EPI_BF16>(gK, wN, a, 1, st); break;
        case 3: e = run_tc<false, true, 192, 4, false, EPI_BF16>(gK, wN, a, 1, st); break;
        default: e = run_tc<false, true, 256, 4, false, EPI_BF16>(gK, wN, a, 1, st); break;
    }
    if (e != cudaSuccess) return e;
    switch ((d.R + 63) / 64) {
        case 2: e = run_tc<true, true, 128, 4, true, EPI_F32_PART>(gM, uN, b, d.splits, st); break;
        case 3: e = run_tc<true, true, 192, 4, true, EPI_F32_PART>(gM, uN, b, d.splits, st); break;
        default: e = run_tc<true, true, 256, 3, true, EPI_F32_PART>(gM, uN, b, d.splits, st); break;
    }
    if (e != cudaSuccess) return e;
    dtp_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(d.part, d.splits, d.D, d.R, d.dw,
                                                                    d.dbias);
    return cudaGetLastError();
}

}  // namespace ssm
