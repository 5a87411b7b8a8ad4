/*
 * ssm_scan.h — C ABI of the B200 selective diagonal state-space scan and its exact gradient.
 *
 * What the calls compute
 * ----------------------
 * Real mode (the selective SSM of "选择性状态空间模型(S3M)原理与工程实践" §1.1: step size
 * delta = softplus(projection), decay A = -exp(log_A), transition exp(A·delta); input term taken
 * as the Euler form delta·B_t·x_t), per batch b and channel d, for states n = 0..N-1:
 *
 *     delta_t = softplus(delta_raw_t)          A_n = -exp(A_log[d,n])
 *     h_t,n   = exp(delta_t A_n) h_{t-1,n} + delta_t Bm_t,n x_t          h_{-1} = 0
 *     y_t     = sum_n Cm_t,n h_t,n + Dskip[d] x_t
 *
 * ssm_scan_bwd returns the exact gradient of sum(dy·y) by a reverse-time adjoint scan ("Breaking
 * the Memory Wall: Exact Analytical Differentiation via Tiled Operator-Space Evolution", abstract:
 * exact analytical derivatives without materialising the graph; tiled operator-space evolution).
 * Only the state at the end of every chunk of T steps is stored (the checkpoint buffer, O(L/T));
 * the backward recomputes each chunk from its checkpoint.  The time-parallel structure (local scan
 * of a chunk, carry across chunks, correction) follows the three-phase scan described for Flash
 * PD-SSM ("Flash PD-SSM", technical summary, hardware-aware implementation, phases A–C).
 *
 * Complex mode ("SPARC: Shared Phase and Retention Control for Efficient Adaptive Spectral
 * Recurrence", abstract: two shared input-dependent scalars drive every complex mode, each mode
 * keeps its own timescale and frequency; diagonal affine recurrence), per batch b and mode k:
 *
 *     s_t = softplus(r_t)      a_t,k = exp(-lambda_k s_t + i omega_k phi_t)
 *     h_t,k = a_t,k h_{t-1,k} + u_t,k                                   h_{-1} = 0
 *
 * and ssm_scan_complex_bwd returns the gradient of Re sum conj(g)·h with respect to u (complex,
 * as d/dRe + i d/dIm), r, phi, lambda and omega, recomputing each chunk from the checkpoints the
 * forward wrote (ssm_scan_complex_bwd_traj computes the same from a stored trajectory h).
 *
 * Conventions (all calls)
 * -----------------------
 * - Every pointer argument is a DEVICE pointer owned by the caller, except the shape structs,
 *   which are host pointers read during the call only.  The library allocates no memory and
 *   keeps no state between calls; calls on different streams with different buffers may overlap.
 * - Arrays are dense row-major (C order), no strides.  Every array pointer must be 16-byte
 *   aligned (SSM_ERR_MISALIGNED otherwise).
 * - Calls enqueue kernels on `stream` and return without synchronising.  Argument errors are
 *   detected on the host before anything is enqueued (nothing is written).  A failed launch
 *   returns SSM_ERR_CUDA.  Conditions found on the device (non-finite state) are recorded in a
 *   status word at the start of the workspace; ssm_scan_status() reads it.  Each fwd/bwd call
 *   resets that word when it starts.
 * - Gradients overwrite their outputs (they do not accumulate).  All outputs are deterministic:
 *   the same inputs give bitwise the same outputs on every run (no floating-point atomics).
 * - Workspace: a caller-owned device buffer of at least ssm_scan_*_workspace_bytes() bytes,
 *   used as scratch by one call at a time (do not share one workspace between overlapping calls).
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSM_SCAN_ABI_VERSION 5  /* 4: complex forward writes checkpoints; checkpointed complex
                                  backward (ssm_scan_complex_bwd); the trajectory-reading one
                                  is ssm_scan_complex_bwd_traj.  5: ssm_scan_options.flags
                                  (was reserved), SSM_FUSED_SUMS */

/* Same underlying type as cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st* ssm_stream_t;

typedef enum ssm_status {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1,          /* null pointer, negative size, reserved field not zero */
    SSM_ERR_UNSUPPORTED = 2,          /* dstate not in {4,8,16}, chunk not in {16..256}, bad io */
    SSM_ERR_MISALIGNED = 3,           /* pointer not 16-byte aligned, or dim*sizeof(io) % 16 != 0 */
    SSM_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes below the size query's answer */
    SSM_ERR_CUDA = 5,                 /* a kernel launch or CUDA runtime call failed */
    SSM_ERR_TIMEOUT = 6,              /* a bounded device-side wait gave up (device-side) */
    SSM_ERR_NONFINITE = 7             /* a NaN or Inf reached a carried state (device-side) */
} ssm_status;

typedef enum ssm_dtype { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

/* Real-mode problem size.  Beyond the sizes the method itself needs (batch, seqlen, dim, dstate,
 * chunk, io) it carries seg_chunks, a performance knob that never changes the result beyond
 * rounding, and a reserved word kept for later fields. */
typedef struct ssm_shape {
    int64_t batch;      /* B >= 0 */
    int64_t seqlen;     /* L >= 0 (0 is a valid empty problem) */
    int64_t dim;        /* D >= 1; D * sizeof(io) must be a multiple of 16 bytes */
    int64_t dstate;     /* N, one of 4, 8, 16 */
    int32_t chunk;      /* T, one of 16, 32, 64, 128, 256: checkpoint spacing in steps */
    int32_t io;         /* ssm_dtype of x, delta_raw, Bm, Cm, y, dy, dx, ddelta_raw, dB, dC */
    int32_t seg_chunks; /* time-parallel split, in chunks per segment; 0 = automatic.  A tuning
                           knob only: results agree to rounding for every value. */
    int32_t reserved;   /* must be 0 */
} ssm_shape;

/* Complex-mode problem size (with the same seg_chunks knob as ssm_shape). */
typedef struct ssm_cshape {
    int64_t batch;      /* B >= 0 */
    int64_t seqlen;     /* L >= 0 */
    int64_t modes;      /* K >= 1, even */
    int32_t chunk;      /* T, one of 16..256: checkpoint spacing and time-split granularity */
    int32_t seg_chunks; /* chunks per time segment; 0 = automatic (tuning knob only) */
} ssm_cshape;

/* ABI version of the loaded library (SSM_SCAN_ABI_VERSION at build time). */
int ssm_scan_abi_version(void);

/* Bytes of the checkpoint buffer: B * ceil(L/T) * D * N * sizeof(float).  Layout
 * [B, ceil(L/T), D, N] fp32; entry c holds h at the last step of chunk c (step min((c+1)T, L)-1).
 * Returns 0 for an invalid shape. */
size_t ssm_scan_checkpoint_bytes(const ssm_shape* shape);

/* Workspace bytes for ssm_scan_fwd (backward == 0) or ssm_scan_bwd (backward != 0); at least
 * 256.  Returns 0 for an invalid shape. */
size_t ssm_scan_workspace_bytes(const ssm_shape* shape, int backward);

/*
 * Forward scan.
 *   x, delta_raw  [B, L, D]  io dtype           Bm, Cm  [B, L, N]  io dtype
 *   A_log         [D, N]     fp32               Dskip   [D]        fp32
 * Outputs:
 *   y             [B, L, D]  io dtype
 *   ckpt          [B, ceil(L/T), D, N] fp32 (ssm_scan_checkpoint_bytes); keep it for the backward
 * Returns an ssm_status.
 */
int ssm_scan_fwd(const ssm_shape* shape,
                 const void* x, const void* delta_raw, const float* A_log,
                 const void* Bm, const void* Cm, const float* Dskip,
                 void* y, float* ckpt,
                 void* ws, size_t ws_bytes, ssm_stream_t stream);

/*
 * Backward: exact gradient of sum(dy * y) for the forward above.
 *   inputs as for ssm_scan_fwd, plus ckpt (written by ssm_scan_fwd on the same inputs) and
 *   dy [B, L, D] io dtype.
 * Outputs (overwritten):
 *   dx, ddelta_raw [B, L, D] io dtype;   dB, dC [B, L, N] io dtype;
 *   dA_log [D, N] fp32;                  dD [D] fp32.
 * Returns an ssm_status.
 */
int ssm_scan_bwd(const ssm_shape* shape,
                 const void* x, const void* delta_raw, const float* A_log,
                 const void* Bm, const void* Cm, const float* Dskip,
                 const float* ckpt, const void* dy,
                 void* dx, void* ddelta_raw, float* dA_log, void* dB, void* dC, float* dD,
                 void* ws, size_t ws_bytes, ssm_stream_t stream);

/* Input-term discretisation.  SSM_EULER: b_t = delta_t B_t x_t (the form used above).
 * SSM_ZOH: zero-order hold, the discretisation B̄ = (delta A)^{-1} (exp(delta A) - 1) delta B of
 * "选择性状态空间模型(S3M)原理与工程实践" §1.1, which for a diagonal A is
 * b_{t,n} = (exp(delta_t A_n) - 1) / A_n * B_{t,n} x_t. */
typedef enum ssm_discretization { SSM_EULER = 0, SSM_ZOH = 1 } ssm_discretization;

/* Options of the real-mode calls (all zero / NULL = the plain calls above).  The pointers are
 * device pointers owned by the caller, [B, D, N] fp32 row-major, 16-byte aligned, or NULL.
 * The forward and the backward of one pair must get the same discretization and h0. */
/* ssm_scan_options.flags.  SSM_FUSED_SUMS (backward): when all CTAs of a backward launch can be
 * resident at once (444 at N = 4 or 8, 592 at N = 16 on a B200), it runs cooperatively and the
 * scan kernel sums the per-CTA dB/dC partial rows itself, each CTA its share of a chunk once the
 * chunk is done in every channel tile of its batch row, and drops the summed rows from L2
 * unwritten: no reduction kernel, and on a B=8, L=2048, D=1536, N=16 bf16 problem 317 instead of
 * 503 MB of DRAM traffic per call, for about 3 % more time.  Same results to rounding (the channel
 * tiles are added in another fixed order; still deterministic).  Launches that cannot be resident
 * at once use the reduction kernel as without the flag. */
#define SSM_FUSED_SUMS 1

typedef struct ssm_scan_options {
    int32_t discretization; /* ssm_discretization */
    int32_t flags;          /* SSM_FUSED_SUMS or 0; other bits must be 0 */
    const float* h0;        /* initial state h_{-1} (NULL: zero); read by forward and backward */
    float* hL;              /* forward: final state h_{L-1} written here (NULL: not written);
                               with L = 0 it is h0 */
    const float* dhL;       /* backward: upstream gradient of hL (NULL: zero); the loss is then
                               sum(dy * y) + sum(dhL * hL) */
    float* dh0;             /* backward: gradient of the loss w.r.t. h0 written here (NULL: not
                               written); with L = 0 it is dhL */
} ssm_scan_options;

/* ssm_scan_fwd with options (opts may be NULL).  Carrying hL of one call into h0 of the next
 * streams a long sequence through several calls with the same result as one call (to rounding).
 * Returns an ssm_status; SSM_ERR_INVALID_ARG for an unknown discretization or flag. */
int ssm_scan_fwd_ex(const ssm_shape* shape, const ssm_scan_options* opts,
                    const void* x, const void* delta_raw, const float* A_log,
                    const void* Bm, const void* Cm, const float* Dskip,
                    void* y, float* ckpt,
                    void* ws, size_t ws_bytes, ssm_stream_t stream);

/* ssm_scan_bwd with options (opts may be NULL): the exact gradient of
 * sum(dy * y) + sum(dhL * hL), plus dh0.  ckpt must come from ssm_scan_fwd_ex with the same
 * discretization and h0.  Workspace as for ssm_scan_bwd. */
int ssm_scan_bwd_ex(const ssm_shape* shape, const ssm_scan_options* opts,
                    const void* x, const void* delta_raw, const float* A_log,
                    const void* Bm, const void* Cm, const float* Dskip,
                    const float* ckpt, const void* dy,
                    void* dx, void* ddelta_raw, float* dA_log, void* dB, void* dC, float* dD,
                    void* ws, size_t ws_bytes, ssm_stream_t stream);

/*
 * Forward scan for callers that cannot allocate device memory (the pages describe no such call;
 * it exists for integrators whose device memory is owned by someone else, or whose code path may
 * not call cudaMalloc).  Same inputs, outputs and results as ssm_scan_fwd, but no workspace
 * argument: the scratch is a fixed 8 MiB array compiled into the library, held on every GPU that
 * loads it until the process exits.
 * - Shapes whose forward workspace (ssm_scan_workspace_bytes(shape, 0)) exceeds 8 MiB are
 *   rejected with SSM_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.  Only problems that
 *   the library splits into many time segments need more than 256 bytes.
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current; make that first call before any stream capture.  The address is kept
 *   for the life of the process: after cudaDeviceReset on a device, do not call this entry point
 *   on that device again (the array may have moved).
 * - Every call on a device shares the one array and leaves its contents behind; calls that
 *   overlap on the GPU (other streams, other host threads) race on it.  Serialise them.
 * - The device status word is kept in that array and is not readable through ssm_scan_status.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
int ssm_scan_fwd_noalloc(const ssm_shape* shape,
                         const void* x, const void* delta_raw, const float* A_log,
                         const void* Bm, const void* Cm, const float* Dskip,
                         void* y, float* ckpt, ssm_stream_t stream);

/* Workspace bytes for the complex calls (at least 256); 0 for an invalid shape.  backward != 0
 * covers both backward calls (the checkpointed one needs the larger workspace: it adds a
 * per-CTA chunk-trajectory scratch capped at max(64 MiB, the checkpoint bytes)). */
size_t ssm_scan_complex_workspace_bytes(const ssm_cshape* shape, int backward);

/* Bytes of the complex checkpoints: B * ceil(L / T) * K * 8 (complex64); 0 for an invalid shape. */
size_t ssm_scan_complex_checkpoint_bytes(const ssm_cshape* shape);

/*
 * Complex forward ("SPARC: Shared Phase and Retention Control for Efficient Adaptive Spectral
 * Recurrence", abstract: two input-dependent scalars shared by every mode, diagonal recurrence):
 *     s_t = softplus(r_t),  a_{t,k} = exp(-lambda_k s_t + i omega_k phi_t),  h_t = a_t h_{t-1} + u_t.
 *   u       [B, L, K] complex64 (interleaved re, im fp32)
 *   r, phi  [B, L] fp32          lambda, omega [K] fp32
 * Outputs (either may be NULL, not both; SSM_ERR_INVALID_ARG when both are):
 *   h       [B, L, K] complex64: the whole state trajectory (the output of this mode)
 *   ckpt    [B, ceil(L/T), K] complex64: the state at the last step of every chunk of T steps,
 *           what ssm_scan_complex_bwd recomputes from
 */
int ssm_scan_complex_fwd(const ssm_cshape* shape,
                         const void* u, const float* r, const float* phi,
                         const float* lambda, const float* omega,
                         void* h, void* ckpt, void* ws, size_t ws_bytes, ssm_stream_t stream);

/*
 * Complex backward from checkpoints: the gradient of Re sum conj(g)·h, where only the chunk-end
 * states are kept ("Breaking the Memory Wall: Exact Analytical Differentiation via Tiled
 * Operator-Space Evolution", abstract).  Each chunk's trajectory is recomputed from its entering
 * checkpoint into an L2-resident workspace region, then the adjoint
 *     mu_t = g_t + conj(a_{t+1}) mu_{t+1},   q_t = mu_t conj(a_t h_{t-1})
 * is swept back through it:  du = mu,  dlambda = -sum s Re q,  dr = sigmoid(r) (-sum_k lambda Re q),
 * domega = sum phi Im q,  dphi = sum_k omega Im q.  The trajectory h need not be kept: memory
 * beyond inputs and outputs is O(L / T).  Every transition is evaluated twice (recompute and
 * sweep), so this is slower than ssm_scan_complex_bwd_traj, which reads a stored h instead.
 *   u       [B, L, K] complex64, the forward's input
 *   r, phi, lambda, omega as for the forward
 *   ckpt    [B, ceil(L/T), K] complex64, written by ssm_scan_complex_fwd with the same shape
 *   g       [B, L, K] complex64 (dLoss/dh)
 * Outputs (overwritten):
 *   du [B, L, K] complex64;  dr, dphi [B, L] fp32;  dlambda, domega [K] fp32.
 * Enqueues ssm_scan_complex_kernel_launches(shape, 1) kernels.  Returns an ssm_status.
 */
int ssm_scan_complex_bwd(const ssm_cshape* shape,
                         const void* u, const float* r, const float* phi,
                         const float* lambda, const float* omega, const void* ckpt,
                         const void* g, void* du, float* dr, float* dphi, float* dlambda,
                         float* domega, void* ws, size_t ws_bytes, ssm_stream_t stream);

/*
 * Complex backward from the stored trajectory (the fast path when h is resident anyway, e.g.
 * because it is this mode's output): the same gradient as ssm_scan_complex_bwd, with h_{t-1}
 * read from h at every step instead of recomputed, so each transition is evaluated once.
 *   h       [B, L, K] complex64, the trajectory written by ssm_scan_complex_fwd
 *   r, phi, lambda, omega, g, outputs as for ssm_scan_complex_bwd.
 * Enqueues ssm_scan_complex_kernel_launches(shape, 2) kernels.  Returns an ssm_status.
 */
int ssm_scan_complex_bwd_traj(const ssm_cshape* shape,
                              const void* h, const float* r, const float* phi,
                              const float* lambda, const float* omega, const void* g,
                              void* du, float* dr, float* dphi, float* dlambda, float* domega,
                              void* ws, size_t ws_bytes, ssm_stream_t stream);

/* Workspace bytes for ssm_scan_complex_rtrl (at least 256); 0 for an invalid shape. */
size_t ssm_scan_complex_rtrl_workspace_bytes(const ssm_cshape* shape);

/*
 * Complex forward with exact structured real-time recurrent learning ("SPARC: Shared Phase and
 * Retention Control for Efficient Adaptive Spectral Recurrence", abstract: the diagonal recurrence
 * supports exact structured RTRL for online credit assignment).  The state's sensitivities to its
 * mode's own parameters travel with it,
 *     S^lambda_t = a_t S^lambda_{t-1} - s_t a_t h_{t-1},   S^omega_t = a_t S^omega_{t-1} + i phi_t a_t h_{t-1},
 * and the gradient of the online loss Re sum_t conj(g_t) h_t accumulates step by step:
 *     dlambda_k = sum_{b,t} Re(conj(g) S^lambda),  domega_k = sum_{b,t} Re(conj(g) S^omega).
 * One forward pass; no reverse sweep; nothing of the trajectory is stored.  The result equals
 * the lambda/omega gradients of ssm_scan_complex_bwd (to rounding).
 *   u, g     [B, L, K] complex64      r, phi [B, L] fp32      lambda, omega [K] fp32
 *   h        [B, L, K] complex64 trajectory out, or NULL (not written)
 *   state    [B, 3, K] complex64 (h, dh/dlambda, dh/domega), or NULL (start from zero, final
 *            values not returned).  When given it is read as the state before the first step and
 *            overwritten with the state after the last, so consecutive calls on consecutive parts
 *            of a sequence continue it; the caller sums their dlambda/domega.
 *   dlambda, domega [K] fp32: this call's sums (overwritten; zero when B or L is 0).
 * shape->chunk must be valid (16..256) but is not used; shape->seg_chunks is ignored (each CTA
 * walks the whole sequence).  Enqueues 2 kernels (none when B or L is 0).  Returns an ssm_status.
 */
int ssm_scan_complex_rtrl(const ssm_cshape* shape,
                          const void* u, const float* r, const float* phi,
                          const float* lambda, const float* omega, const void* g,
                          void* h, void* state, float* dlambda, float* domega,
                          void* ws, size_t ws_bytes, ssm_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Flash PD-SSM ("Flash PD-SSM: Memory-Optimized Structured Sparse State-Space Models",
 * technical summary: hard selection, gradient propagation).  Per batch b and head e a real state
 * h in R^N; at every step one of K dictionary matrices is chosen by the step's scores and
 * multiplied by a diagonal:
 *     k_t = argmax_k scores[b,t,e,k]   (ties: the lowest k)
 *     h_t = P_{k_t} D_t h_{t-1} + bt_t,   D_t = diag(d[b,t,e,:]),   h_{-1} = h0 (NULL: zero)
 * P_k is a one-hot column selector: column j holds a single 1, in row dict[k*N + j] (several
 * columns may share a row).  Layout: scores [B,L,H,K], d, bt, h, g, dd, dbt [B,L,H,N] fp32,
 * dict [K,N] int32 (entries in [0, N); an entry out of range is clamped and sets
 * SSM_ERR_INVALID_ARG in the workspace status word), sel [B,L,H] int32, h0, dh0 [B,H,N] fp32.
 */
typedef struct ssm_pdshape {
    int64_t batch;   /* B >= 0 */
    int64_t seqlen;  /* L >= 0 */
    int64_t heads;   /* H >= 1, at most 2^21 */
    int32_t nstate;  /* N, one of 4, 8, 16, 32 */
    int32_t ndict;   /* K, 1..32 */
    int32_t reserved; /* must be 0 */
    int32_t reserved2; /* must be 0 */
} ssm_pdshape;

/* Workspace bytes of the PD-SSM calls (the status word: 256); 0 for an invalid shape. */
size_t ssm_pdssm_workspace_bytes(const ssm_pdshape* shape);

/* Forward: writes the trajectory h and the selection sel (argmax of the scores, lowest index on
 * ties).  Enqueues ssm_pdssm_kernel_launches(shape, 0) kernels.  Returns an ssm_status. */
int ssm_pdssm_fwd(const ssm_pdshape* shape, const float* scores, const int32_t* dict,
                  const float* d, const float* bt, const float* h0, float* h, int32_t* sel,
                  void* ws, size_t ws_bytes, ssm_stream_t stream);

/* Backward of L = sum_t <g_t, h_t> for the forward above (h and sel as it wrote them).  The
 * adjoint runs through the hard forward matrices,
 *     mu_t = g_t + A_{t+1}^T mu_{t+1},   (A^T mu)_j = d_j mu[dict[k*N + j]],
 *     dbt = mu,   dd_t[j] = mu_t[dict[k_t*N + j]] h_{t-1}[j],   dh0 = A_0^T mu_0 (dh0 may be NULL),
 * and the discrete selection gets the straight-through surrogate with temperature tau > 0
 * (hard in the forward pass, softmax(scores / tau) in the backward pass):
 *     c_k = <mu_t, P_k D_t h_{t-1}>,   dscores_t[k] = p_k (c_k - sum_k' p_k' c_k') / tau.
 * Enqueues ssm_pdssm_kernel_launches(shape, 1) kernels.  Returns an ssm_status. */
int ssm_pdssm_bwd(const ssm_pdshape* shape, float tau, const float* scores, const int32_t* dict,
                  const float* d, const float* h0, const float* h, const int32_t* sel,
                  const float* g, float* dd, float* dbt, float* dscores, float* dh0,
                  void* ws, size_t ws_bytes, ssm_stream_t stream);

/*
 * Step-size projection in front of the real scan ("选择性状态空间模型(S3M)原理与工程实践" §1.1:
 * delta = softplus(projection(x)); §4.1 merges the discretisation with this matrix product).  One
 * row m per (batch, step); each row's low-rank input u[m, :] maps to the pre-activation of every
 * channel:
 *     delta_raw[m, d] = sum_r u[m, r] w[d, r] + bias[d]
 * which ssm_scan_fwd / ssm_scan_bwd then take as delta_raw ([B, L, D] is [M, D] with M = B*L).
 * The backward of L for an upstream g = dL/d delta_raw (ssm_scan_bwd's ddelta_raw):
 *     du[m, r] = sum_d g[m, d] w[d, r],   dw[d, r] = sum_m g[m, d] u[m, r],   dbias[d] = sum_m g[m, d].
 * Tensor-core GEMMs with bf16 operands and fp32 accumulation; delta_raw and du are rounded to bf16
 * once, dw and dbias are fp32.  Layout: u, du [M, R], w [D, R], delta_raw, g [M, D] bf16;
 * bias, dbias [D], dw [D, R] fp32; bias and dbias may be NULL.  The kernels wait on their
 * tensor-core work through bounded waits; one that gives up writes no output and records
 * SSM_ERR_TIMEOUT in the workspace status word (ssm_scan_status reads it; each call resets it).
 */
typedef struct ssm_dtshape {
    int64_t rows;   /* M >= 0 (0 is a valid empty problem), at most 65535 * 128 */
    int64_t dim;    /* D, a multiple of 8 in 8..2^22 */
    int32_t rank;   /* R, a multiple of 16 in 16..256 */
    int32_t io;     /* SSM_BF16 (the only supported I/O type: SSM_ERR_UNSUPPORTED otherwise) */
} ssm_dtshape;

/* Workspace bytes of ssm_dtproj_fwd (backward == 0: the 256-byte status word) or ssm_dtproj_bwd
 * (backward != 0: the status word, then fp32 partial sums of dw and dbias over splits of 1024
 * rows, ceil(M / 1024) * D * (R + 1) * 4 bytes rounded up to 256); 0 for an invalid shape. */
size_t ssm_dtproj_workspace_bytes(const ssm_dtshape* shape, int backward);

/* delta_raw = u w^T + bias.  Enqueues 1 kernel.  ws: caller-owned device workspace of at least
 * ssm_dtproj_workspace_bytes(shape, 0) bytes, 16-byte aligned.  Returns an ssm_status. */
int ssm_dtproj_fwd(const ssm_dtshape* shape, const void* u, const void* w, const float* bias,
                   void* delta_raw, void* ws, size_t ws_bytes, ssm_stream_t stream);

/* du, dw, dbias for g = dL/d delta_raw.  Enqueues 3 kernels (du; dw and dbias partial sums;
 * their fixed-order reduction).  ws: at least ssm_dtproj_workspace_bytes(shape, 1) bytes.
 * Returns an ssm_status. */
int ssm_dtproj_bwd(const ssm_dtshape* shape, const void* u, const void* w, const void* g,
                   void* du, float* dw, float* dbias, void* ws, size_t ws_bytes,
                   ssm_stream_t stream);

/* Number of kernels one ssm_scan_fwd (backward == 0) / ssm_scan_bwd (backward == 1) call
 * enqueues for this shape (0 for an empty problem, -1 for an invalid shape); backward == 2 counts
 * a backward with SSM_FUSED_SUMS on a device that holds 444 of its CTAs at once (592 for N = 16),
 * where each launch whose CTAs all fit drops its reduction kernel. */
int ssm_scan_kernel_launches(const ssm_shape* shape, int backward);

/* Same for the complex calls: backward = 0 ssm_scan_complex_fwd, 1 ssm_scan_complex_bwd (from
 * checkpoints), 2 ssm_scan_complex_bwd_traj (-1 for any other value). */
int ssm_scan_complex_kernel_launches(const ssm_cshape* shape, int backward);

/* Same for the PD-SSM calls: 1 (one scan kernel, with the argmax fused into the forward and the
 * score gradient into the backward), +2 when the sequence is cut into time segments (segment
 * summaries and carry), +1 when ndict * (128 / nstate) > 256 (argmax or score gradient as a
 * kernel of its own). */
int ssm_pdssm_kernel_launches(const ssm_pdshape* shape, int backward);

/* Waits for `stream`, then returns the status word the last call on `ws` left (SSM_OK,
 * SSM_ERR_NONFINITE or SSM_ERR_TIMEOUT), or SSM_ERR_CUDA if the copy itself fails. */
int ssm_scan_status(const void* ws, ssm_stream_t stream);

/* Static, human-readable name of a status code. */
const char* ssm_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
