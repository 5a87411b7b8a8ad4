// C-ABI entry points (include/ssm_scan.h): argument validation on the host, workspace layout,
// kernel launches.  Nothing here allocates memory or keeps state between calls.
#include "../../include/ssm_scan.h"
#include "ssm_internal.h"

#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr size_t kStatusBytes = 256;
// The real backward keeps its scratch-slot mask in the status block, after the status word:
// (kStatusBytes - kSlotMaskOffset) * 8 = 1984 slots at most.
constexpr size_t kSlotMaskOffset = 32;
constexpr int kTargetCtas = 296;  // 2 x 148 SMs: below this many CTAs, split time into segments
// Real forward, once split: enough segments for about 2368 CTAs (two waves at the eight CTAs per
// SM its registers and shared memory allow), so that every SM keeps several CTAs busy.
constexpr int64_t kRealFwdSplitCtas = 2368;
// Real backward: 4 CTAs per SM (126 registers per thread, 48 KB of shared memory) on 148 SMs.
// Also the number of scratch slots (window-start states, (delta, sigma)) of a launch with more
// CTAs: a CTA holds one from its start to its end.
constexpr int64_t kRealBwdSlots = 592;

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool valid_chunk(int T) { return T == 16 || T == 32 || T == 64 || T == 128 || T == 256; }

// Time segments of a forward: none when ctas_per_seg reaches kTargetCtas, else enough for about
// `split_ctas` CTAs in all.
int pick_segments(int64_t ctas_per_seg, int nC, int forced, int64_t split_ctas, int* seg_chunks) {
    if (nC <= 0) {
        *seg_chunks = 1;
        return 1;
    }
    int sc;
    if (forced > 0) {
        sc = forced < nC ? forced : nC;
    } else {
        int64_t nseg = 1;
        if (ctas_per_seg < kTargetCtas) nseg = (split_ctas + ctas_per_seg - 1) / ctas_per_seg;
        if (nseg > nC) nseg = nC;
        sc = (int)((nC + nseg - 1) / nseg);
    }
    *seg_chunks = sc;
    return (nC + sc - 1) / sc;
}

struct RealPlan {
    int B, L, D, N, T, nC, ndt, seg_chunks, nseg, esz;
    // backward: its own segmentation (see real_bwd_impl): b_nseg segments of b_seg_chunks
    // chunks, concurrent (b_seq = 0, b_group per launch) or sequential blocks (b_seq = 1)
    int b_nseg, b_seg_chunks, b_seq, b_group, b_rows, b_launches;
    // workspace offsets (bytes); fwd and bwd use separate layouts
    size_t f_sumP, f_sumS, f_hin, f_end;
    size_t b_gP, b_gG, b_part, b_dA, b_dD, b_bnd, b_cnt, b_end;
    int b_nslot;  // backward scratch slots: CTAs per launch, at most the resident CTAs
};

int plan_real(const ssm_shape* s, RealPlan* p) {
    if (!s) return SSM_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0 || s->dim < 1 || s->reserved != 0 || s->seg_chunks < 0)
        return SSM_ERR_INVALID_ARG;
    if (s->dstate != 4 && s->dstate != 8 && s->dstate != 16) return SSM_ERR_UNSUPPORTED;
    if (!valid_chunk(s->chunk)) return SSM_ERR_UNSUPPORTED;
    if (s->io != SSM_F32 && s->io != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    // index arithmetic inside the kernels is 32-bit for per-row offsets and grid sizes
    if (s->batch > 65535 || s->seqlen > (int64_t)1 << 30 || s->dim > (int64_t)1 << 24)
        return SSM_ERR_UNSUPPORTED;
    p->esz = s->io == SSM_BF16 ? 2 : 4;
    if ((s->dim * p->esz) % 16 != 0) return SSM_ERR_MISALIGNED;
    p->B = (int)s->batch;
    p->L = (int)s->seqlen;
    p->D = (int)s->dim;
    p->N = (int)s->dstate;
    p->T = s->chunk;
    p->nC = (p->L + p->T - 1) / p->T;
    const int DT = ssm::real_dt(p->N);
    p->ndt = (p->D + DT - 1) / DT;
    p->nseg = pick_segments((int64_t)p->B * p->ndt, p->nC, s->seg_chunks, kRealFwdSplitCtas,
                            &p->seg_chunks);
    if (p->nseg > 65535) return SSM_ERR_UNSUPPORTED;

    const size_t B = p->B, DN = (size_t)p->D * p->N, S = p->nseg;
    size_t o = kStatusBytes;
    const size_t summ = S > 1 ? B * (S - 1) * DN * 4 : 0;
    p->f_sumP = o; o = align256(o + summ);
    p->f_sumS = o; o = align256(o + summ);
    p->f_hin = o;  o = align256(o + (S > 1 ? B * S * DN * 4 : 0));
    p->f_end = o;

    // Backward.  The per-CTA dB/dC partial sums cover the steps of one launch; time is walked
    // in launches whose partial buffer fits max(half the checkpoint bytes, 128 MiB), so the
    // backward's memory stays O(L / T) however long the sequence.
    const size_t per_chunk = (size_t)p->ndt * B * p->T * 2 * p->N * 4;
    const size_t ckpt = B * (size_t)p->nC * DN * 4;
    const size_t cap = ckpt / 2 > ((size_t)128 << 20) ? ckpt / 2 : ((size_t)128 << 20);
    const int64_t ctas_per_seg = (int64_t)B * p->ndt;
    const size_t chunks_cap = per_chunk > 0 ? cap / per_chunk : (size_t)p->nC;  // per launch
    const int nC1 = p->nC > 0 ? p->nC : 1;
    auto clampi = [](size_t v, size_t lo, size_t hi) { return (int)(v < lo ? lo : (v > hi ? hi : v)); };
    // launches as large as the partial-sum cap allows: the scratch is one slot per resident CTA
    const size_t segs_cap = (size_t)p->nC + 1;
    // one wave of CTAs (kTargetCtas..kRealBwdSlots), or several waves that fill the SMs to at
    // least 80 %: no time split.  Otherwise (too few CTAs, or a partial last wave that would
    // leave most SMs idle) concurrent segments of at most 4 chunks, each launch holding as many
    // segments as the caps allow.
    const int64_t waves = (ctas_per_seg + kRealBwdSlots - 1) / kRealBwdSlots;
    const bool fill = ctas_per_seg >= kTargetCtas &&
                      (ctas_per_seg <= kRealBwdSlots || 5 * ctas_per_seg >= 4 * waves * kRealBwdSlots);
    if (s->seg_chunks > 0) {
        // forced time split: concurrent segments, as many per launch as the caps allow
        p->b_seg_chunks = s->seg_chunks < nC1 ? s->seg_chunks : nC1;
        p->b_nseg = (nC1 + p->b_seg_chunks - 1) / p->b_seg_chunks;
        p->b_seq = 0;
        const size_t g = chunks_cap / p->b_seg_chunks;
        p->b_group = clampi(g < segs_cap ? g : segs_cap, 1, p->b_nseg);
    } else if (fill || nC1 <= 1) {
        // no time split: one pass, or sequential blocks if the partial sums of the whole
        // sequence would exceed the cap
        if (chunks_cap >= (size_t)nC1) {
            p->b_nseg = 1;
            p->b_seg_chunks = nC1;
            p->b_seq = 0;
        } else {
            p->b_seg_chunks = clampi(chunks_cap, 1, nC1);
            p->b_nseg = (nC1 + p->b_seg_chunks - 1) / p->b_seg_chunks;
            p->b_seq = 1;
        }
        p->b_group = 1;
    } else {
        // concurrent segments of 4 chunks when there are at least 2 x 4 CTA-chunks of work per
        // CTA slot (the summary pass then stays a small share of the work), shorter for smaller
        // problems so that more of them run at once; launches of equal size
        const int64_t work = (int64_t)nC1 * ctas_per_seg / (2 * kRealBwdSlots);
        p->b_seg_chunks = (int)(work < 1 ? 1 : (work > 4 ? 4 : work));
        if (p->b_seg_chunks > nC1) p->b_seg_chunks = nC1;
        p->b_nseg = (nC1 + p->b_seg_chunks - 1) / p->b_seg_chunks;
        p->b_seq = 0;
        const size_t g = chunks_cap / p->b_seg_chunks;
        const int gmax = clampi(g < segs_cap ? g : segs_cap, 1, p->b_nseg);
        const int nl = (p->b_nseg + gmax - 1) / gmax;
        p->b_group = (p->b_nseg + nl - 1) / nl;
    }
    if (p->b_nseg > 65535) return SSM_ERR_UNSUPPORTED;
    const size_t BS = p->b_nseg;
    const int per = p->b_seq ? 1 : p->b_group;
    p->b_launches = (p->b_nseg + per - 1) / per;
    const size_t rows = (size_t)per * p->b_seg_chunks * p->T;
    p->b_rows = (int)(rows < (size_t)p->L ? rows : (size_t)p->L);
    // gG holds the summaries' local adjoints and then, overwritten by the carry, the adjoint
    // entering each segment but the last (sequential blocks hand it over through gG too)
    const size_t bvin = BS > 1 ? B * (BS - 1) * DN * 4 : 0;
    // gP (the summaries' products) is dead once the carry has run, before any scan CTA writes its
    // dA_log partial sum: the two share one region
    o = kStatusBytes;
    p->b_gP = o;   o = align256(o + B * BS * DN * 4);
    p->b_dA = p->b_gP;
    p->b_gG = o;   o = align256(o + bvin);
    p->b_part = o; o = align256(o + (size_t)p->ndt * B * (size_t)p->b_rows * 2 * p->N * 4);
    p->b_dD = o;   o = align256(o + B * BS * (size_t)p->D * 4);
    const int64_t ctas = (int64_t)p->ndt * p->B * per;
    p->b_nslot = (int)(ctas < kRealBwdSlots ? (ctas > 0 ? ctas : 1) : kRealBwdSlots);
    p->b_bnd = o;  o = align256(o + (size_t)p->b_nslot * ssm::real_bwd_scratch_floats(p->N, p->T) * 4);
    p->b_cnt = o;  o = align256(o + BS * B * 4);  // chunks finished per (segment, batch row)
    p->b_end = o;
    return SSM_OK;
}

struct CplxPlan {
    int B, L, K, T, nC, nkt, seg_chunks, nseg;
    int b_group;  // checkpointed backward: segments per launch (the trajectory scratch holds one)
    size_t f_sumP, f_sumS, f_hin, f_end;
    size_t b_gP, b_gG, b_win, b_rp, b_lo, b_traj, b_end;
    size_t r_lo, r_end;  // RTRL: per-(batch, mode) gradient sums
};

// Checkpointed complex backward: per-launch cap on the chunk-trajectory scratch
// (max(checkpoint bytes, this)), so the backward's memory stays O(L / T).
constexpr size_t kCplxTrajCap = (size_t)64 << 20;

int plan_cplx(const ssm_cshape* s, CplxPlan* p) {
    if (!s) return SSM_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0 || s->modes < 1 || s->seg_chunks < 0)
        return SSM_ERR_INVALID_ARG;
    if (!valid_chunk(s->chunk)) return SSM_ERR_UNSUPPORTED;
    if (s->batch > 65535 || s->seqlen > (int64_t)1 << 30 || s->modes > (int64_t)1 << 26)
        return SSM_ERR_UNSUPPORTED;
    if (s->modes % 2 != 0) return SSM_ERR_MISALIGNED;
    p->B = (int)s->batch;
    p->L = (int)s->seqlen;
    p->K = (int)s->modes;
    p->T = s->chunk;
    p->nC = (p->L + p->T - 1) / p->T;
    p->nkt = (p->K + ssm::kCplxKT - 1) / ssm::kCplxKT;
    p->nseg = pick_segments((int64_t)p->B * p->nkt, p->nC, s->seg_chunks, kTargetCtas, &p->seg_chunks);
    if (p->nseg > 65535) return SSM_ERR_UNSUPPORTED;
    const size_t B = p->B, K = p->K, S = p->nseg;
    const size_t summ = S > 1 ? B * (S - 1) * K * 8 : 0;
    size_t o = kStatusBytes;
    p->f_sumP = o; o = align256(o + summ);
    p->f_sumS = o; o = align256(o + summ);
    p->f_hin = o;  o = align256(o + (S > 1 ? B * S * K * 8 : 0));
    p->f_end = o;
    o = kStatusBytes;
    p->b_gP = o;  o = align256(o + summ);
    p->b_gG = o;  o = align256(o + summ);
    p->b_win = o; o = align256(o + (S > 1 ? B * S * K * 8 : 0));
    p->b_rp = o;  o = align256(o + (size_t)p->nkt * B * (size_t)p->L * 8);
    p->b_lo = o;  o = align256(o + B * S * K * 8);
    // checkpointed backward: [group][B][nkt] CTAs' chunk trajectories
    const size_t traj_seg = B * (size_t)p->nkt * ssm::cplx_traj_floats(p->T) * 4;
    const size_t ckpt = B * (size_t)p->nC * K * 8;
    const size_t cap = ckpt > kCplxTrajCap ? ckpt : kCplxTrajCap;
    const size_t g = traj_seg > 0 ? cap / traj_seg : S;
    p->b_group = (int)(g < 1 ? 1 : (g > S ? S : g));
    p->b_traj = o; o = align256(o + (size_t)p->b_group * traj_seg);
    p->b_end = o;
    o = kStatusBytes;
    p->r_lo = o;  o = align256(o + B * K * 8);
    p->r_end = o;
    return SSM_OK;
}

// A pointer may be null only when the array it describes is empty.
bool ptr_ok(const void* ptr, size_t count) { return count == 0 || ptr != nullptr; }

int check_arrays(const void* const* ptrs, const size_t* counts, int n) {
    for (int i = 0; i < n; ++i) {
        if (!ptr_ok(ptrs[i], counts[i])) return SSM_ERR_INVALID_ARG;
        if (counts[i] && !aligned16(ptrs[i])) return SSM_ERR_MISALIGNED;
    }
    return SSM_OK;
}

int check_options(const ssm_scan_options& o) {
    if ((o.flags & ~SSM_FUSED_SUMS) != 0) return SSM_ERR_INVALID_ARG;
    if (o.discretization != SSM_EULER && o.discretization != SSM_ZOH) return SSM_ERR_INVALID_ARG;
    return SSM_OK;
}

// dst <- src (n floats), or zeros when src is null; nothing when dst is null.
int copy_or_zero(float* dst, const float* src, size_t n, cudaStream_t s) {
    if (!dst || n == 0) return SSM_OK;
    const cudaError_t e = src ? cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(dst, 0, n * sizeof(float), s);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace

extern "C" {

int ssm_scan_abi_version(void) { return SSM_SCAN_ABI_VERSION; }

size_t ssm_scan_checkpoint_bytes(const ssm_shape* shape) {
    RealPlan p;
    if (plan_real(shape, &p) != SSM_OK) return 0;
    return (size_t)p.B * p.nC * p.D * p.N * sizeof(float);
}

size_t ssm_scan_workspace_bytes(const ssm_shape* shape, int backward) {
    RealPlan p;
    if (plan_real(shape, &p) != SSM_OK) return 0;
    return backward ? p.b_end : p.f_end;
}

int ssm_scan_fwd_ex(const ssm_shape* shape, const ssm_scan_options* opts, const void* x,
                    const void* delta_raw, const float* A_log, const void* Bm, const void* Cm,
                    const float* Dskip, void* y, float* ckpt, void* ws, size_t ws_bytes,
                    ssm_stream_t stream) {
    RealPlan p;
    int st = plan_real(shape, &p);
    if (st != SSM_OK) return st;
    const ssm_scan_options o = opts ? *opts : ssm_scan_options{};
    if ((st = check_options(o)) != SSM_OK) return st;
    const size_t BLD = (size_t)p.B * p.L * p.D, BLN = (size_t)p.B * p.L * p.N;
    const size_t DN = (size_t)p.D * p.N, ck = (size_t)p.B * p.nC * DN, BDN = (size_t)p.B * DN;
    const void* ptrs[] = {x, delta_raw, A_log, Bm, Cm, Dskip, y, ckpt, ws, o.h0, o.hL};
    const size_t counts[] = {BLD, BLD, DN, BLN, BLN, (size_t)p.D, BLD, ck, 1,
                             o.h0 ? BDN : 0, o.hL ? BDN : 0};
    if ((st = check_arrays(ptrs, counts, 11)) != SSM_OK) return st;
    if (ws_bytes < p.f_end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (p.B == 0) return SSM_OK;
    if (p.L == 0)  // the final state is the initial one
        return copy_or_zero(o.hL, o.h0, BDN, s);
    ssm::RealArgs a = {};
    a.B = p.B; a.L = p.L; a.D = p.D; a.T = p.T; a.nC = p.nC;
    a.seg_chunks = p.seg_chunks; a.nseg = p.nseg; a.ndt = p.ndt;
    a.x = x; a.draw = delta_raw; a.A_log = A_log; a.Bm = Bm; a.Cm = Cm; a.Dskip = Dskip;
    a.y = y; a.ckpt = ckpt;
    a.sumP = at<float>(ws, p.f_sumP); a.sumS = at<float>(ws, p.f_sumS); a.hin = at<float>(ws, p.f_hin);
    a.status = at<unsigned>(ws, 0);
    a.h0 = o.h0; a.hL = o.hL; a.zoh = o.discretization == SSM_ZOH;
    return ssm::launch_real_fwd(a, shape->io == SSM_BF16, p.N, s) == cudaSuccess ? SSM_OK
                                                                                : SSM_ERR_CUDA;
}

int ssm_scan_fwd(const ssm_shape* shape, const void* x, const void* delta_raw, const float* A_log,
                 const void* Bm, const void* Cm, const float* Dskip, void* y, float* ckpt, void* ws,
                 size_t ws_bytes, ssm_stream_t stream) {
    return ssm_scan_fwd_ex(shape, nullptr, x, delta_raw, A_log, Bm, Cm, Dskip, y, ckpt, ws,
                           ws_bytes, stream);
}

int ssm_scan_bwd_ex(const ssm_shape* shape, const ssm_scan_options* opts, const void* x,
                    const void* delta_raw, const float* A_log, const void* Bm, const void* Cm,
                    const float* Dskip, const float* ckpt, const void* dy, void* dx,
                    void* ddelta_raw, float* dA_log, void* dB, void* dC, float* dD, void* ws,
                    size_t ws_bytes, ssm_stream_t stream) {
    RealPlan p;
    int st = plan_real(shape, &p);
    if (st != SSM_OK) return st;
    const ssm_scan_options o = opts ? *opts : ssm_scan_options{};
    if ((st = check_options(o)) != SSM_OK) return st;
    const size_t BLD = (size_t)p.B * p.L * p.D, BLN = (size_t)p.B * p.L * p.N;
    const size_t DN = (size_t)p.D * p.N, ck = (size_t)p.B * p.nC * DN, BDN = (size_t)p.B * DN;
    const void* ptrs[] = {x, delta_raw, A_log, Bm, Cm, Dskip, ckpt, dy,
                          dx, ddelta_raw, dA_log, dB, dC, dD, ws, o.h0, o.dhL, o.dh0};
    const size_t counts[] = {BLD, BLD, DN, BLN, BLN, (size_t)p.D, ck, BLD,
                             BLD, BLD, DN, BLN, BLN, (size_t)p.D, 1,
                             o.h0 ? BDN : 0, o.dhL ? BDN : 0, o.dh0 ? BDN : 0};
    if ((st = check_arrays(ptrs, counts, 18)) != SSM_OK) return st;
    if (ws_bytes < p.b_end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // status word and scratch-slot mask; the chunk counters of the fused dB/dC sums when asked for
    if (cudaMemsetAsync(ws, 0, kStatusBytes, s) != cudaSuccess) return SSM_ERR_CUDA;
    if ((o.flags & SSM_FUSED_SUMS) && p.B > 0 && p.L > 0 &&
        cudaMemsetAsync(at<unsigned char>(ws, p.b_cnt), 0, (size_t)p.b_nseg * p.B * 4, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (p.B == 0 || p.L == 0) {
        if (cudaMemsetAsync(dA_log, 0, DN * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        if (cudaMemsetAsync(dD, 0, (size_t)p.D * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        return copy_or_zero(o.dh0, o.dhL, BDN, s);  // with no steps, dL/dh0 = dL/dhL
    }
    ssm::RealArgs a = {};
    a.B = p.B; a.L = p.L; a.D = p.D; a.T = p.T; a.nC = p.nC;
    a.seg_chunks = p.b_seg_chunks; a.nseg = p.b_nseg; a.ndt = p.ndt;
    a.seq_blocks = p.b_seq; a.part_rows = p.b_rows;
    a.x = x; a.draw = delta_raw; a.A_log = A_log; a.Bm = Bm; a.Cm = Cm; a.Dskip = Dskip;
    a.ckpt_in = ckpt; a.dy = dy; a.dx = dx; a.ddraw = ddelta_raw;
    a.gsumP = at<float>(ws, p.b_gP); a.gsumG = at<float>(ws, p.b_gG); a.vin = a.gsumG;
    a.dBC_part = at<float>(ws, p.b_part); a.dA_part = at<float>(ws, p.b_dA);
    a.dD_part = at<float>(ws, p.b_dD);
    a.bnd_scratch = at<float>(ws, p.b_bnd);
    a.slot_mask = at<unsigned>(ws, kSlotMaskOffset);
    a.nslot = p.b_nslot;
    a.grp_cnt = at<unsigned>(ws, p.b_cnt);
    a.fused_sums = (o.flags & SSM_FUSED_SUMS) != 0;
    a.dB = dB; a.dC = dC; a.dA_log = dA_log; a.dD = dD;
    a.status = at<unsigned>(ws, 0);
    a.h0 = o.h0; a.dhL = o.dhL; a.dh0 = o.dh0; a.zoh = o.discretization == SSM_ZOH;
    return ssm::launch_real_bwd(a, shape->io == SSM_BF16, p.N, p.b_group, s) == cudaSuccess
               ? SSM_OK
               : SSM_ERR_CUDA;
}

int ssm_scan_bwd(const ssm_shape* shape, const void* x, const void* delta_raw, const float* A_log,
                 const void* Bm, const void* Cm, const float* Dskip, const float* ckpt,
                 const void* dy, void* dx, void* ddelta_raw, float* dA_log, void* dB, void* dC,
                 float* dD, void* ws, size_t ws_bytes, ssm_stream_t stream) {
    return ssm_scan_bwd_ex(shape, nullptr, x, delta_raw, A_log, Bm, Cm, Dskip, ckpt, dy, dx,
                           ddelta_raw, dA_log, dB, dC, dD, ws, ws_bytes, stream);
}

int ssm_scan_kernel_launches(const ssm_shape* shape, int backward) {
    RealPlan p;
    if (plan_real(shape, &p) != SSM_OK) return -1;
    if (p.B == 0 || p.L == 0) return 0;
    if (!backward) return p.nseg > 1 ? 3 : 1;  // [segment summary + carry] + scan
    // [summary + carry] + per launch (main + dB/dC reduce) + dA_log/dD reduce; with
    // SSM_FUSED_SUMS (backward == 2) no reduce for a launch whose CTAs are all resident at once
    // on 148 SMs (3 per SM, 4 for the N = 16 instance)
    int n = (p.b_nseg > 1 && !p.b_seq ? 2 : 0) + 1;
    const int per = p.b_seq ? 1 : p.b_group;
    for (int hi = p.b_nseg; hi > 0; hi -= per) {
        const int segs = hi - per > 0 ? per : hi;
        const int64_t ctas = (int64_t)p.ndt * p.B * segs;
        const int64_t resident = p.N == 16 ? kRealBwdSlots : 444;
        n += (backward == 2 && ctas <= p.b_nslot && ctas <= resident) ? 1 : 2;
    }
    return n;
}

int ssm_scan_complex_kernel_launches(const ssm_cshape* shape, int backward) {
    CplxPlan p;
    if (plan_cplx(shape, &p) != SSM_OK || backward < 0 || backward > 2) return -1;
    if (p.B == 0 || p.L == 0) return 0;
    const int seg = p.nseg > 1 ? 2 : 0;
    if (backward == 1) return seg + (p.nseg + p.b_group - 1) / p.b_group + 2;
    return backward ? 3 + seg : 1 + seg;
}

size_t ssm_scan_complex_checkpoint_bytes(const ssm_cshape* shape) {
    CplxPlan p;
    if (plan_cplx(shape, &p) != SSM_OK) return 0;
    return (size_t)p.B * p.nC * p.K * 8;
}

size_t ssm_scan_complex_workspace_bytes(const ssm_cshape* shape, int backward) {
    CplxPlan p;
    if (plan_cplx(shape, &p) != SSM_OK) return 0;
    return backward ? p.b_end : p.f_end;
}

int ssm_scan_complex_fwd(const ssm_cshape* shape, const void* u, const float* r, const float* phi,
                         const float* lambda, const float* omega, void* h, void* ckpt, void* ws,
                         size_t ws_bytes, ssm_stream_t stream) {
    CplxPlan p;
    int st = plan_cplx(shape, &p);
    if (st != SSM_OK) return st;
    const size_t BLK = (size_t)p.B * p.L * p.K, BL = (size_t)p.B * p.L;
    const size_t CK = (size_t)p.B * p.nC * p.K;
    if (!h && !ckpt) return SSM_ERR_INVALID_ARG;  // nothing to write
    const void* ptrs[] = {u, r, phi, lambda, omega, h, ckpt, ws};
    const size_t counts[] = {BLK, BL, BL, (size_t)p.K, (size_t)p.K, h ? BLK : 0, ckpt ? CK : 0, 1};
    if ((st = check_arrays(ptrs, counts, 8)) != SSM_OK) return st;
    if (ws_bytes < p.f_end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (p.B == 0 || p.L == 0) return SSM_OK;
    ssm::CplxArgs a = {};
    a.B = p.B; a.L = p.L; a.K = p.K; a.T = p.T; a.nC = p.nC;
    a.seg_chunks = p.seg_chunks; a.nseg = p.nseg; a.nkt = p.nkt;
    a.u = static_cast<const float*>(u); a.r = r; a.phi = phi; a.lam = lambda; a.om = omega;
    a.h = static_cast<float*>(h);
    a.ckpt = static_cast<float*>(ckpt);
    a.sumP = at<float>(ws, p.f_sumP); a.sumS = at<float>(ws, p.f_sumS); a.hin = at<float>(ws, p.f_hin);
    a.status = at<unsigned>(ws, 0);
    return ssm::launch_cplx_fwd(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

size_t ssm_scan_complex_rtrl_workspace_bytes(const ssm_cshape* shape) {
    CplxPlan p;
    if (plan_cplx(shape, &p) != SSM_OK) return 0;
    return p.r_end;
}

int ssm_scan_complex_rtrl(const ssm_cshape* shape, const void* u, const float* r,
                          const float* phi, const float* lambda, const float* omega, const void* g,
                          void* h, void* state, float* dlambda, float* domega, void* ws,
                          size_t ws_bytes, ssm_stream_t stream) {
    CplxPlan p;
    int st = plan_cplx(shape, &p);
    if (st != SSM_OK) return st;
    const size_t BLK = (size_t)p.B * p.L * p.K, BL = (size_t)p.B * p.L;
    const void* ptrs[] = {u, r, phi, lambda, omega, g, dlambda, domega, ws, h, state};
    const size_t counts[] = {BLK, BL, BL, (size_t)p.K, (size_t)p.K, BLK, (size_t)p.K, (size_t)p.K,
                             1, h ? BLK : 0, state ? (size_t)p.B * 3 * p.K : 0};
    if ((st = check_arrays(ptrs, counts, 11)) != SSM_OK) return st;
    if (ws_bytes < p.r_end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (p.B == 0 || p.L == 0) {  // no steps: no gradient, the state is unchanged
        if (cudaMemsetAsync(dlambda, 0, (size_t)p.K * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        if (cudaMemsetAsync(domega, 0, (size_t)p.K * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        return SSM_OK;
    }
    ssm::CplxArgs a = {};
    a.B = p.B; a.L = p.L; a.K = p.K; a.T = p.T; a.nC = p.nC;
    a.seg_chunks = p.nC; a.nseg = 1; a.nkt = p.nkt;
    a.u = static_cast<const float*>(u); a.r = r; a.phi = phi; a.lam = lambda; a.om = omega;
    a.g = static_cast<const float*>(g);
    a.h = static_cast<float*>(h);
    a.state = static_cast<float*>(state);
    a.lo_part = at<float>(ws, p.r_lo);
    a.dlam = dlambda; a.dom = domega;
    a.status = at<unsigned>(ws, 0);
    return ssm::launch_cplx_rtrl(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_scan_complex_bwd(const ssm_cshape* shape, const void* u, const float* r, const float* phi,
                         const float* lambda, const float* omega, const void* ckpt, const void* g,
                         void* du, float* dr, float* dphi, float* dlambda, float* domega, void* ws,
                         size_t ws_bytes, ssm_stream_t stream) {
    CplxPlan p;
    int st = plan_cplx(shape, &p);
    if (st != SSM_OK) return st;
    const size_t BLK = (size_t)p.B * p.L * p.K, BL = (size_t)p.B * p.L, K = p.K;
    const size_t CK = (size_t)p.B * p.nC * p.K;
    const void* ptrs[] = {u, r, phi, lambda, omega, ckpt, g, du, dr, dphi, dlambda, domega, ws};
    const size_t counts[] = {BLK, BL, BL, K, K, CK, BLK, BLK, BL, BL, K, K, 1};
    if ((st = check_arrays(ptrs, counts, 13)) != SSM_OK) return st;
    if (ws_bytes < p.b_end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (p.B == 0 || p.L == 0) {
        if (cudaMemsetAsync(dlambda, 0, K * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        if (cudaMemsetAsync(domega, 0, K * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        return SSM_OK;
    }
    ssm::CplxArgs a = {};
    a.B = p.B; a.L = p.L; a.K = p.K; a.T = p.T; a.nC = p.nC;
    a.seg_chunks = p.seg_chunks; a.nseg = p.nseg; a.nkt = p.nkt;
    a.u = static_cast<const float*>(u); a.r = r; a.phi = phi; a.lam = lambda; a.om = omega;
    a.ckpt_in = static_cast<const float*>(ckpt); a.g = static_cast<const float*>(g);
    a.du = static_cast<float*>(du); a.dr = dr; a.dphi = dphi; a.dlam = dlambda; a.dom = domega;
    a.gsumP = at<float>(ws, p.b_gP); a.gsumG = at<float>(ws, p.b_gG); a.win = at<float>(ws, p.b_win);
    a.rp_part = at<float>(ws, p.b_rp); a.lo_part = at<float>(ws, p.b_lo);
    a.traj = at<float>(ws, p.b_traj);
    a.status = at<unsigned>(ws, 0);
    return ssm::launch_cplx_bwd_ckpt(a, p.b_group, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_scan_complex_bwd_traj(const ssm_cshape* shape, const void* h, const float* r,
                              const float* phi, const float* lambda, const float* omega,
                              const void* g, void* du, float* dr, float* dphi, float* dlambda,
                              float* domega, void* ws, size_t ws_bytes, ssm_stream_t stream) {
    CplxPlan p;
    int st = plan_cplx(shape, &p);
    if (st != SSM_OK) return st;
    const size_t BLK = (size_t)p.B * p.L * p.K, BL = (size_t)p.B * p.L, K = p.K;
    const void* ptrs[] = {h, r, phi, lambda, omega, g, du, dr, dphi, dlambda, domega, ws};
    const size_t counts[] = {BLK, BL, BL, K, K, BLK, BLK, BL, BL, K, K, 1};
    if ((st = check_arrays(ptrs, counts, 12)) != SSM_OK) return st;
    if (ws_bytes < p.b_end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (p.B == 0 || p.L == 0) {
        if (cudaMemsetAsync(dlambda, 0, K * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        if (cudaMemsetAsync(domega, 0, K * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        return SSM_OK;
    }
    ssm::CplxArgs a = {};
    a.B = p.B; a.L = p.L; a.K = p.K; a.T = p.T; a.nC = p.nC;
    a.seg_chunks = p.seg_chunks; a.nseg = p.nseg; a.nkt = p.nkt;
    a.r = r; a.phi = phi; a.lam = lambda; a.om = omega;
    a.h_in = static_cast<const float*>(h); a.g = static_cast<const float*>(g);
    a.du = static_cast<float*>(du); a.dr = dr; a.dphi = dphi; a.dlam = dlambda; a.dom = domega;
    a.gsumP = at<float>(ws, p.b_gP); a.gsumG = at<float>(ws, p.b_gG); a.win = at<float>(ws, p.b_win);
    a.rp_part = at<float>(ws, p.b_rp); a.lo_part = at<float>(ws, p.b_lo);
    a.status = at<unsigned>(ws, 0);
    return ssm::launch_cplx_bwd(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// ------------------------------------------------------------------------------ Flash PD-SSM
namespace {
int check_pdshape(const ssm_pdshape* s) {
    if (!s) return SSM_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0 || s->heads < 1 || s->reserved != 0 || s->reserved2 != 0)
        return SSM_ERR_INVALID_ARG;
    if (s->nstate != 4 && s->nstate != 8 && s->nstate != 16 && s->nstate != 32) return SSM_ERR_UNSUPPORTED;
    if (s->ndict < 1 || s->ndict > 32) return SSM_ERR_UNSUPPORTED;
    if (s->batch > 65535 || s->seqlen > (int64_t)1 << 30 || s->heads > (int64_t)1 << 21 ||
        (double)s->batch * s->seqlen * s->heads * s->nstate > 9.0e15)
        return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

// Time segments of the PD-SSM scans: when the (batch, head-group) CTAs are fewer than kPdMinCtas
// (each streams at most a few tens of GB/s, bounded by its per-step latency), the sequence is cut
// into segments of a multiple of 16 steps (at least 64) so that about four CTAs per SM run; the
// workspace holds their summaries and carries.
constexpr int64_t kPdMinCtas = 128;

struct PdPlan {
    int nseg, seg_len;
    size_t f_pi, f_w, f_s, hin, b_rho, b_v, b_w, win, end;
};

PdPlan plan_pd(const ssm_pdshape* s) {
    PdPlan p = {};
    const int64_t B = s->batch, L = s->seqlen, H = s->heads, N = s->nstate;
    const int64_t seq = ssm::kPdThreads / N, ctas = B * ((H + seq - 1) / seq);
    int64_t nseg = 1;
    if (ctas > 0 && ctas < kPdMinCtas && L >= 128) {
        nseg = (2 * kTargetCtas + ctas - 1) / ctas;
        nseg = nseg < L / 64 ? nseg : L / 64;
        if (nseg < 1) nseg = 1;
    }
    int64_t seg_len = (L + nseg - 1) / nseg;
    seg_len = (seg_len + 15) / 16 * 16;
    if (seg_len < 16) seg_len = 16;
    nseg = L > 0 ? (L + seg_len - 1) / seg_len : 1;
    p.nseg = (int)nseg;
    p.seg_len = (int)seg_len;
    const size_t BHN = (size_t)B * H * N, S = (size_t)nseg;
    const size_t summ = S > 1 ? BHN * (S - 1) * 4 : 0, carry = S > 1 ? BHN * S * 4 : 0;
    size_t o = kStatusBytes;
    p.f_pi = o;  o = align256(o + summ);
    p.f_w = o;   o = align256(o + summ);
    p.f_s = o;   o = align256(o + summ);
    p.hin = o;   o = align256(o + carry);
    p.b_rho = o; o = align256(o + summ);
    p.b_v = o;   o = align256(o + summ);
    p.b_w = o;   o = align256(o + summ);
    p.win = o;   o = align256(o + carry);
    p.end = o;
    return p;
}

ssm::PdArgs pd_args(const ssm_pdshape* s, void* ws) {
    ssm::PdArgs a = {};
    a.B = (int)s->batch; a.L = (int)s->seqlen; a.H = (int)s->heads; a.N = s->nstate; a.K = s->ndict;
    a.status = at<unsigned>(ws, 0);
    const PdPlan p = plan_pd(s);
    a.nseg = p.nseg; a.seg_len = p.seg_len;
    a.f_pi = at<int32_t>(ws, p.f_pi); a.f_w = at<float>(ws, p.f_w); a.f_s = at<float>(ws, p.f_s);
    a.hin = at<float>(ws, p.hin);
    a.b_rho = at<int32_t>(ws, p.b_rho); a.b_v = at<float>(ws, p.b_v); a.b_w = at<float>(ws, p.b_w);
    a.win = at<float>(ws, p.win);
    return a;
}
}  // namespace

int ssm_pdssm_kernel_launches(const ssm_pdshape* shape, int backward) {
    (void)backward;  // the forward and the backward launch the same number
    if (check_pdshape(shape) != SSM_OK) return -1;
    if (shape->batch == 0 || shape->seqlen == 0) return 0;
    return ssm::pdssm_launches(pd_args(shape, nullptr));
}

size_t ssm_pdssm_workspace_bytes(const ssm_pdshape* shape) {
    return check_pdshape(shape) == SSM_OK ? plan_pd(shape).end : 0;
}

int ssm_pdssm_fwd(const ssm_pdshape* shape, const float* scores, const int32_t* dict,
                  const float* d, const float* bt, const float* h0, float* h, int32_t* sel,
                  void* ws, size_t ws_bytes, ssm_stream_t stream) {
    int st = check_pdshape(shape);
    if (st != SSM_OK) return st;
    const size_t BLH = (size_t)shape->batch * shape->seqlen * shape->heads;
    const size_t N = shape->nstate, K = shape->ndict, BH = (size_t)shape->batch * shape->heads;
    const void* ptrs[] = {scores, dict, d, bt, h, sel, ws, h0};
    const size_t counts[] = {BLH * K, K * N, BLH * N, BLH * N, BLH * N, BLH, 1, h0 ? BH * N : 0};
    if ((st = check_arrays(ptrs, counts, 8)) != SSM_OK) return st;
    if (ws_bytes < plan_pd(shape).end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (BLH == 0) return SSM_OK;
    ssm::PdArgs a = pd_args(shape, ws);
    a.scores = scores; a.dict = dict; a.d = d; a.bt = bt; a.h0 = h0; a.h = h; a.sel = sel;
    return ssm::launch_pdssm_fwd(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_pdssm_bwd(const ssm_pdshape* shape, float tau, const float* scores, const int32_t* dict,
                  const float* d, const float* h0, const float* h, const int32_t* sel,
                  const float* g, float* dd, float* dbt, float* dscores, float* dh0, void* ws,
                  size_t ws_bytes, ssm_stream_t stream) {
    int st = check_pdshape(shape);
    if (st != SSM_OK) return st;
    if (!(tau > 0.0f && tau < 3.0e38f)) return SSM_ERR_INVALID_ARG;
    const size_t BLH = (size_t)shape->batch * shape->seqlen * shape->heads;
    const size_t N = shape->nstate, K = shape->ndict, BH = (size_t)shape->batch * shape->heads;
    const void* ptrs[] = {scores, dict, d, h, sel, g, dd, dbt, dscores, ws, h0, dh0};
    const size_t counts[] = {BLH * K, K * N, BLH * N, BLH * N, BLH, BLH * N, BLH * N, BLH * N,
                             BLH * K, 1, h0 ? BH * N : 0, dh0 ? BH * N : 0};
    if ((st = check_arrays(ptrs, counts, 12)) != SSM_OK) return st;
    if (ws_bytes < plan_pd(shape).end) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (BLH == 0) {  // no steps: dL/dh0 = 0
        if (dh0 && BH && cudaMemsetAsync(dh0, 0, BH * N * sizeof(float), s) != cudaSuccess)
            return SSM_ERR_CUDA;
        return SSM_OK;
    }
    ssm::PdArgs a = pd_args(shape, ws);
    a.tau = tau; a.scores = scores; a.dict = dict; a.d = d; a.h0 = h0;
    a.h = const_cast<float*>(h); a.sel = const_cast<int32_t*>(sel); a.g = g;
    a.dd = dd; a.dbt = dbt; a.dscores = dscores; a.dh0 = dh0;
    return ssm::launch_pdssm_bwd(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

namespace {
int check_dtshape(const ssm_dtshape* s) {
    if (!s) return SSM_ERR_INVALID_ARG;
    if (s->rows < 0 || s->dim < 1 || s->rank < 1) return SSM_ERR_INVALID_ARG;
    if (s->io != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    if (s->dim % 8 != 0 || s->dim < 8 || s->rank % 16 != 0 || s->rank > 256) return SSM_ERR_UNSUPPORTED;
    if (s->rows > (int64_t)65535 * 128 || s->dim > ((int64_t)1 << 22)) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

int dt_splits(const ssm_dtshape* s) {
    const int64_t k = ssm::dtproj_rows_per_split(s->rank);
    return (int)((s->rows + k - 1) / k);
}
}  // namespace

size_t ssm_dtproj_workspace_bytes(const ssm_dtshape* shape, int backward) {
    if (check_dtshape(shape) != SSM_OK) return 0;
    if (!backward) return kStatusBytes;
    const size_t b = (size_t)dt_splits(shape) * shape->dim * (shape->rank + 1) * sizeof(float);
    return kStatusBytes + align256(b);
}

int ssm_dtproj_fwd(const ssm_dtshape* shape, const void* u, const void* w, const float* bias,
                   void* delta_raw, void* ws, size_t ws_bytes, ssm_stream_t stream) {
    int st = check_dtshape(shape);
    if (st != SSM_OK) return st;
    const size_t M = shape->rows, D = shape->dim, R = shape->rank;
    const void* ptrs[] = {u, w, delta_raw, ws, bias};
    const size_t counts[] = {M * R, D * R, M * D, 1, bias ? D : 0};
    if ((st = check_arrays(ptrs, counts, 5)) != SSM_OK) return st;
    if (ws_bytes < ssm_dtproj_workspace_bytes(shape, 0)) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (M == 0) return SSM_OK;
    ssm::DtArgs a = {};
    a.M = (int64_t)M; a.D = (int64_t)D; a.R = (int)R;
    a.u = u; a.w = w; a.bias = bias; a.delta_raw = delta_raw;
    a.status = at<unsigned>(ws, 0);
    return ssm::launch_dtproj_fwd(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_dtproj_bwd(const ssm_dtshape* shape, const void* u, const void* w, const void* g,
                   void* du, float* dw, float* dbias, void* ws, size_t ws_bytes,
                   ssm_stream_t stream) {
    int st = check_dtshape(shape);
    if (st != SSM_OK) return st;
    const size_t M = shape->rows, D = shape->dim, R = shape->rank;
    const void* ptrs[] = {u, w, g, du, dw, ws, dbias};
    const size_t counts[] = {M * R, D * R, M * D, M * R, D * R, 1, dbias ? D : 0};
    if ((st = check_arrays(ptrs, counts, 7)) != SSM_OK) return st;
    if (ws_bytes < ssm_dtproj_workspace_bytes(shape, 1)) return SSM_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (M == 0) {  // no rows: the sums are empty
        if (cudaMemsetAsync(dw, 0, D * R * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        if (dbias && cudaMemsetAsync(dbias, 0, D * sizeof(float), s) != cudaSuccess) return SSM_ERR_CUDA;
        return SSM_OK;
    }
    ssm::DtArgs a = {};
    a.M = (int64_t)M; a.D = (int64_t)D; a.R = (int)R; a.splits = dt_splits(shape);
    a.u = u; a.w = w; a.g = g; a.du = du; a.dw = dw; a.dbias = dbias;
    a.part = at<float>(ws, kStatusBytes);
    a.status = at<unsigned>(ws, 0);
    return ssm::launch_dtproj_bwd(a, s) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_scan_status(const void* ws, ssm_stream_t stream) {
    if (!ws) return SSM_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SSM_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSM_ERR_CUDA;
    return (int)v;
}

const char* ssm_status_string(int status) {
    switch (status) {
        case SSM_OK: return "SSM_OK";
        case SSM_ERR_INVALID_ARG: return "SSM_ERR_INVALID_ARG: null pointer, negative size or nonzero reserved field";
        case SSM_ERR_UNSUPPORTED: return "SSM_ERR_UNSUPPORTED: dstate, chunk, io dtype or size outside the supported set";
        case SSM_ERR_MISALIGNED: return "SSM_ERR_MISALIGNED: pointer not 16-byte aligned or row not a multiple of 16 bytes";
        case SSM_ERR_WORKSPACE_TOO_SMALL: return "SSM_ERR_WORKSPACE_TOO_SMALL: workspace below the size query's answer";
        case SSM_ERR_CUDA: return "SSM_ERR_CUDA: a CUDA launch or runtime call failed";
        case SSM_ERR_TIMEOUT: return "SSM_ERR_TIMEOUT: a bounded device-side wait gave up";
        case SSM_ERR_NONFINITE: return "SSM_ERR_NONFINITE: a NaN or Inf reached a carried state";
        default: return "unknown ssm_status";
    }
}

}  // extern "C"
