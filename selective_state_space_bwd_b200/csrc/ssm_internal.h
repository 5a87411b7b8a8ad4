// Internal (host + device) declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

// Real-mode kernels: a thread owns 4 consecutive states of one channel, N / 4 adjacent lanes
// cover a channel and a CTA covers kRealDT channels of one batch row.
constexpr int kRealDT = 32;

inline int real_dt(int) { return kRealDT; }

// Backward scratch per CTA (floats): the state at every 4-step window start of one chunk
// ([T/4][threads][4]) and (delta, sigmoid(delta_raw)) of one chunk ([T][32] float2).
__host__ __device__ inline size_t real_bwd_scratch_floats(int N, int T) {
    return (size_t)T * (kRealDT * (N / 4)) + (size_t)T * kRealDT * 2;
}

// Complex mode: one thread per mode, kCplxKT modes per CTA, kCplxTT steps staged per tile.
constexpr int kCplxKT = 64;
constexpr int kCplxTT = 32;

struct RealArgs {
    int B, L, D, T, nC, seg_chunks, nseg, ndt;
    const void* x;
    const void* draw;
    const float* A_log;
    const void* Bm;
    const void* Cm;
    const float* Dskip;
    void* y;
    float* ckpt;
    const float* ckpt_in;
    const void* dy;
    void* dx;
    void* ddraw;
    float* sumP;      // forward segment summaries [B][nseg-1][D][N] (segments 0..nseg-2)
    float* sumS;
    float* hin;       // state entering each segment [B][nseg][D][N]
    float* gsumP;     // backward segment summaries [B][nseg-1][D][N] (segments 1..nseg-1)
    float* gsumG;
    float* vin;       // scaled adjoint a_{t+1} g_{t+1} entering segments 0..nseg-2 from their
                      // ends, [B][nseg-1][D][N]; the same buffer as gsumG (the carry overwrites
                      // each summary with it); the last segment takes dhL
    float* dBC_part;  // [ndt][B][part_rows][2N] per-CTA sums over its channels (dB then dC),
                      // rows relative to part_t0 (the first step of the current launch)
    float* dA_part;   // [B][nseg][D][N] sum over the segment of delta * q
    float* dD_part;   // [B][nseg][D]
    float* bnd_scratch;  // backward scratch (L2-resident): nslot slots of real_bwd_scratch_floats,
                         // each held by one resident CTA at a time
    unsigned* slot_mask; // bit i set while slot i is held; zero when a launch starts and ends
    int nslot;
    unsigned* grp_cnt;   // backward, fused dB/dC sums: chunks finished per (segment, batch row)
                         // [nseg][B], zero when the call starts
    int fused_sums;      // backward: SSM_FUSED_SUMS asked for
    int seg0;         // backward: first segment handled by this launch (blockIdx.z offset)
    int seq_blocks;   // backward: segments run as sequential launches, each handing its
                      // entering adjoint to the next through vin
    int part_t0, part_rows;
    void* dB;
    void* dC;
    float* dA_log;
    float* dD;
    unsigned* status;
    // options: initial state h0 and final state hL ([B][D][N] fp32, may be null); upstream
    // gradient dhL of the final state and gradient dh0 of the initial state (backward, may be null);
    // zoh != 0 selects the zero-order-hold input term
    const float* h0;
    float* hL;
    const float* dhL;
    float* dh0;
    int zoh;
};

struct CplxArgs {
    int B, L, K, T, nC, seg_chunks, nseg, nkt;
    const float* u;     // interleaved complex [B][L][K][2]
    const float* r;
    const float* phi;
    const float* lam;
    const float* om;
    float* h;
    const float* h_in;  // trajectory read by the backward
    const float* g;
    float* du;
    float* dr;
    float* dphi;
    float* dlam;
    float* dom;
    float* sumP;        // [B][nseg-1][K][2] forward segment summaries (segments 0..nseg-2)
    float* sumS;
    float* hin;         // [B][nseg][K][2]
    float* gsumP;       // [B][nseg-1][K][2] backward summaries (segments 1..nseg-1)
    float* gsumG;
    float* win;         // [B][nseg][K][2] adjoint entering each segment from its end
    float* rp_part;     // [nkt][B][L][2] per-CTA sums of lambda*Re q and omega*Im q
    float* lo_part;     // [B][nseg][K][2] per-segment sums of -s Re q and phi Im q
    float* state;       // RTRL: [B][3][K][2] (h, dh/dlambda, dh/domega) carried across calls, or null
    unsigned* status;
    // checkpoints: the state at the last step of every chunk, [B][nC][K][2].  The forward writes
    // them when ckpt is not null; the checkpointed backward reads ckpt_in and recomputes each
    // chunk's trajectory into a per-CTA scratch region of cplx_traj_floats(T) floats (L2-resident),
    // running segments [seg0, seg0 + gridDim.z) per launch
    float* ckpt;
    const float* ckpt_in;
    float* traj;
    int seg0;
};
// Floats of one CTA's chunk-trajectory scratch in the checkpointed complex backward.
__host__ __device__ inline size_t cplx_traj_floats(int T) { return (size_t)T * kCplxKT * 2; }

// Flash PD-SSM: N lanes per (batch, head) sequence (lane = state), kPdThreads per CTA.
constexpr int kPdThreads = 128;

struct PdArgs {
    int B, L, H, N, K;
    float tau;
    const float* scores;   // [B][L][H][K]
    const int32_t* dict;   // [K][N]: row of the single 1 in column j of dictionary matrix k
    const float* d;        // [B][L][H][N]
    const float* bt;       // [B][L][H][N]
    const float* h0;       // [B][H][N] or null
    float* h;              // forward: trajectory out; backward: trajectory in
    int32_t* sel;          // forward: selection out; backward: in
    const float* g;        // backward: dL/dh [B][L][H][N]
    float* dd;
    float* dbt;            // backward: also the adjoint mu read by the score-gradient kernel
    float* dscores;
    float* dh0;
    unsigned* status;
    // time segments (the three phases: local scans with composed maps, carry, rescan)
    int nseg, seg_len;
    int32_t* f_pi;  // forward summaries of segments 0..nseg-2 [B*H][nseg-1][N]: map of the
    float* f_w;     //   composed transition (column j -> row f_pi, weight f_w) and local end state
    float* f_s;
    float* hin;     // state entering each segment [B*H][nseg][N]
    int32_t* b_rho; // backward summaries of segments 1..nseg-1 [B*H][nseg-1][N]: composed
    float* b_v;     //   transposed transitions (gather from b_rho, weight b_v) and local adjoint
    float* b_w;
    float* win;     // adjoint entering each segment from its end [B*H][nseg][N]
};

// Step-size projection (csrc/dtproj.cu): bf16 u [M, R], w [D, R], delta_raw / g [M, D],
// du [M, R]; fp32 bias, dw [D, R], dbias [D]; part: `splits` x D x (R+1) fp32 partial sums.
struct DtArgs {
    int64_t M, D;
    int R, splits;
    const void* u;
    const void* w;
    const float* bias;
    void* delta_raw;
    const void* g;
    void* du;
    float* dw;
    float* dbias;
    float* part;
    unsigned* status;  // workspace status word (SSM_ERR_TIMEOUT when a bounded wait gave up)
};
int64_t dtproj_rows_per_split(int R);
cudaError_t launch_dtproj_fwd(const DtArgs& a, cudaStream_t st);
cudaError_t launch_dtproj_bwd(const DtArgs& a, cudaStream_t st);

// Launchers (return cudaGetLastError() of the last launch).
cudaError_t launch_pdssm_fwd(const PdArgs& a, cudaStream_t st);
cudaError_t launch_pdssm_bwd(const PdArgs& a, cudaStream_t st);
int pdssm_launches(const PdArgs& a);  // kernels per ssm_pdssm_fwd (and per ssm_pdssm_bwd) call
cudaError_t launch_real_fwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st);
cudaError_t launch_real_bwd(const RealArgs& a, int io_bf16, int N, int group, cudaStream_t st);
cudaError_t launch_cplx_fwd(const CplxArgs& a, cudaStream_t st);
cudaError_t launch_cplx_rtrl(const CplxArgs& a, cudaStream_t st);
cudaError_t launch_cplx_bwd(const CplxArgs& a, cudaStream_t st);
// checkpointed backward: segments in launches of `group` (the trajectory scratch holds one launch)
cudaError_t launch_cplx_bwd_ckpt(const CplxArgs& a, int group, cudaStream_t st);

}  // namespace ssm
