// Internal (host + device) declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

// Thread layout of the real-mode kernels: every thread owns S consecutive states of one channel
// (S = 4 or 8 for N = 16), NG = N / S adjacent lanes cover a channel, a CTA covers DT = 32
// channels with 32 * NG threads.  The backward holds a window of TS steps of (a_t, a_t h_{t-1})
// per state in registers (TS * S = 32) and parks the state at every window start in an
// L2-resident scratch region of the workspace.
constexpr int kRealDT = 32;
constexpr int kRealMaxTB = 128;  // longest stretch of steps the backward stages at once
constexpr int kRealStates16 = 4;
constexpr int kRealStates8 = 4;

inline int real_dt(int) { return kRealDT; }
inline int real_states(int N) { return N == 16 ? kRealStates16 : (N == 8 ? kRealStates8 : 4); }
inline int real_threads(int N) { return kRealDT * (N / real_states(N)); }
inline int real_window(int N) { return real_states(N) == 4 ? 8 : 4; }
inline size_t real_bnd_floats_per_cta(int N) {
    return (size_t)(kRealMaxTB / real_window(N)) * real_threads(N) * real_states(N);
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
    float* vin;       // scaled adjoint a_{t+1} g_{t+1} entering each segment from its end
    float* dBC_part;  // [ndt][B][L][2N] per-CTA sums over its channels (dB then dC)
    float* dA_part;   // [B][nseg][D][N] sum over the segment of delta * q
    float* dD_part;   // [B][nseg][D]
    float* bnd_scratch;  // per-CTA window-start states of the backward (L2-resident)
    void* dB;
    void* dC;
    float* dA_log;
    float* dD;
    unsigned* status;
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
    unsigned* status;
};

// Launchers (return cudaGetLastError() of the last launch).
cudaError_t launch_real_fwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st);
cudaError_t launch_real_bwd(const RealArgs& a, int io_bf16, int N, cudaStream_t st);
cudaError_t launch_cplx_fwd(const CplxArgs& a, cudaStream_t st);
cudaError_t launch_cplx_bwd(const CplxArgs& a, cudaStream_t st);

}  // namespace ssm
