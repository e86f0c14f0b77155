/*
 * m3.h -- C ABI of the B200 (sm_100a) Mamba-3 selective-scan library.
 *
 * The operation (restated from the pages this library follows; see the
 * citations on each entry point):
 *
 *   alpha_t = exp(dt_t A_h)            beta_t = (1 - lam_t) dt_t alpha_t
 *   gamma_t = lam_t dt_t
 *   Phi_t   = Phi_{t-1} + dt_t theta_t          (per rotation pair i < K)
 *   Bbar_t  = R(Phi_t) B_t,  Cbar_t = R(Phi_t) C_t   (pairs (2i, 2i+1), i < K;
 *                                                     elements 2K.. pass through)
 *   U_t     = Bbar_t x_t^T                      (N x P)
 *   h_t     = alpha_t h_{t-1} + beta_t U_{t-1} + gamma_t U_t
 *   y_t     = Cbar_t^T h_t + D_h x_t
 *
 * with R(phi) the rotation [[cos, -sin], [sin, cos]] of each adjacent pair,
 * h_{-1} = h0, U_{-1} = prev_Bx0, Phi_{-1} = angle0 (zero when NULL).
 *
 * Layouts: row-major, last index fastest, all buffers contiguous.
 *   x, y        (batch, seqlen, nheads, headdim)         M3_F32 or M3_BF16
 *   B, C        (batch, seqlen, ngroups, dstate)         same dtype as x
 *               (batch, seqlen, ngroups, rank, dstate)   MIMO
 *   dt, lam     (batch, seqlen, nheads)                  fp32, post-activation
 *                                                        (dt > 0, 0 <= lam <= 1)
 *   theta       (batch, seqlen, nheads, K)               fp32
 *   A, D        (nheads)                                 fp32
 *   W_x, W_y    (nheads, rank, headdim)                  fp32 (MIMO)
 *   h, prev_Bx  (batch, nheads, dstate, headdim)         fp32
 *   angle       (batch, nheads, K)                       fp32
 * G = ngroups B/C groups (TorchMamba README, "Models": n_groups, with
 * nheads % G == 0): head h reads the B/C row of group h / (nheads / G).
 * K = rotated pairs (partial RoPE; dotLLM pull request, real-checkpoint run:
 * num_rope_angles 32 of dstate 128).  Defaults G = nheads, K = dstate/2.
 *
 * Ownership and execution: the caller owns every buffer (device memory,
 * including the workspace).  The library never allocates, frees or
 * synchronises; every call validates its arguments on the host, then
 * enqueues its kernels on `stream` (a cudaStream_t; NULL = legacy default
 * stream) and returns.  Device pointers must be 16-byte aligned.  Outputs
 * must not alias inputs, except where an entry point says in/out.
 *
 * Errors: validation happens before any launch; on an error nothing is
 * enqueued and no output is written.  A failed launch returns M3_ERR_CUDA.
 * No C++ exception crosses this boundary and there is no fallback path.
 */
#ifndef M3_H
#define M3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    M3_OK = 0,
    M3_ERR_INVALID_ARG = 1,  /* null required pointer, bad size, odd dstate, misalignment */
    M3_ERR_UNSUPPORTED = 2,  /* valid but outside this build's limits (see m3_limits)    */
    M3_ERR_WORKSPACE = 3,    /* workspace missing or smaller than m3_workspace_bytes()   */
    M3_ERR_CUDA = 4,         /* a kernel launch failed                                   */
    M3_ERR_TIMEOUT = 5       /* a bounded wait inside a kernel gave up (m3_device_error) */
} m3_status;

typedef enum { M3_F32 = 0, M3_BF16 = 1 } m3_dtype;

/* Problem sizes.  rank is ignored by the SISO entry points (taken as 1);
 * chunk is the chunk length of the chunked algorithm (>= 1; a request of
 * 2^30 or more behaves as 2^30); seqlen is ignored by the decode steps.
 * ngroups: B/C groups G (0 = nheads; else nheads % ngroups == 0).
 * rope_pairs: rotated pairs K (0 = dstate/2; else 1 <= K <= dstate/2).
 * Anything else is M3_ERR_INVALID_ARG. */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, rank, chunk;
    int64_t ngroups, rope_pairs;
} m3_dims;

/* Optional QkNorm + BC-bias applied to B and C before the rotation
 * (dotLLM pull request, "Key findings": bias after QkNorm, before RoPE):
 *   B <- B / sqrt(mean_n B^2 + eps) * normw_B   (when normw_B != NULL)
 *   B <- B + bias_B[h, r, :]                    (when bias_B  != NULL)
 * and the same for C.  normw_* are (dstate) fp32, bias_* are
 * (nheads, rank, dstate) fp32 (rank = 1 for SISO).  A NULL m3_bcnorm
 * pointer turns both off. */
typedef struct {
    const float *normw_B, *normw_C, *bias_B, *bias_C;
    float eps;
} m3_bcnorm;

/* Limits of this build: dstate <= 256 and even, headdim <= 256,
 * dstate * headdim <= 16384, rank <= 8 (MIMO); batch <= 2^24, nheads <= 4096,
 * batch * nheads <= 2^31 - 1 lanes, and batch * seqlen * nheads *
 * max(headdim, dstate) <= 2^46.  Sizes past them are M3_ERR_UNSUPPORTED. */
typedef struct {
    int64_t max_dstate, max_headdim, max_state_elems, max_rank;
} m3_limits;
m3_limits m3_get_limits(void);

/* S1 -- trapezoidal discretization.  (dotLLM pull request, "Stage A:
 * Mamba3Discretize"; TorchMamba README, "Math notes": exponential-trapezoidal
 * 3-term recurrence, Prop. 1 Eqs. 5-6.)
 * In: dt, lam (batch, seqlen, nheads) fp32; A (nheads) fp32.
 * Out: alpha, beta, gamma (batch, seqlen, nheads) fp32.
 * Uses d.batch, d.seqlen, d.nheads. */
m3_status m3_discretize(const float *dt, const float *A, const float *lam, m3_dims d,
                        float *alpha, float *beta, float *gamma, void *stream);

/* S2 -- QkNorm + BC-bias + data-dependent RoPE.  (dotLLM pull request,
 * "Stage A: Mamba3QkNorm, Mamba3DataRoPE"; TorchMamba README, "Math notes":
 * accumulated data-dependent pairwise rotations, Props. 2-4.)
 * In: B, C (batch, seqlen, ngroups, [rank,] dstate) of `dtype` (rank axis
 * present when d.rank > 1); theta, dt; angle0 (batch, nheads, K) or NULL for
 * zeros; norm or NULL.
 * Out: B_rot, C_rot (batch, seqlen, nheads, [rank,] dstate), one row per
 * head, dtype of B (values rotated in fp32 and rounded to nearest-even on
 * store); angle_final (batch, nheads, K) or NULL.  Every rank uses the same
 * angle. */
m3_status m3_rope_bc(const void *B, const void *C, m3_dtype dtype, const float *theta,
                     const float *dt, const float *angle0, const m3_bcnorm *norm,
                     m3_dims d, void *B_rot, void *C_rot, float *angle_final,
                     void *stream);

/* S1+S2+S3 -- SISO chunked forward of the whole scan.  (dotLLM pull
 * request, "Stage A: Mamba3SelectiveScan", trapezoidal scan Eq. 9 with the
 * prev_Bx second state, and the streaming-decode comment: shifted_gamma and
 * the boundary fold; TorchMamba README, "Math notes": Mamba-2 chunkwise
 * intra-chunk quadratic part plus inter-chunk carry.)
 * In: x, B, C of `dtype`; dt, lam, theta, A, D fp32; h0, prevBx0
 * (batch, nheads, dstate, headdim) and angle0, each NULL for zeros.
 * Out: y (dtype of x), h_final and prevBx_final (fp32, the state after the
 * last token: h_{T-1} and U_{T-1}), angle_final (fp32); the three state
 * outputs may be NULL when not wanted.  When seqlen == 0 the states pass
 * through unchanged.
 * workspace: device scratch of at least m3_workspace_bytes(M3_WS_SISO, d,
 * dtype) bytes (may be NULL when that is 0); its contents on entry do not
 * matter and are undefined on return. */
m3_status m3_siso_chunked_fwd(const void *x, const float *dt, const float *A,
                              const float *lam, const float *theta, const void *B,
                              const void *C, const float *D, m3_dtype dtype,
                              const m3_bcnorm *norm, const float *h0,
                              const float *prevBx0, const float *angle0, m3_dims d,
                              void *y, float *h_final, float *prevBx_final,
                              float *angle_final, void *workspace, size_t workspace_bytes,
                              void *stream);

/* S4 -- rank-R MIMO chunked forward on a shared (dstate, headdim) state.
 * (TorchMamba README, "Models" and "Math notes": rank-R update on a shared
 * (N,P) state, R^2 SISO calls, App. C per-head expand/contract vectors;
 * dotLLM pull request, "Mamba-3 MIMO streaming decode": the state is summed
 * over ranks and the angle is rank-free.)
 *   X_{t,r}[p] = W_x[h,r,p] x_t[p]
 *   U_t        = sum_r Bbar_{t,r} X_{t,r}^T
 *   y_t[p]     = sum_r W_y[h,r,p] (Cbar_{t,r}^T h_t)[p] + D_h x_t[p]
 * Arguments as m3_siso_chunked_fwd plus W_x, W_y (nheads, rank, headdim)
 * fp32, each NULL for all ones; B, C are (batch, seqlen, ngroups, rank,
 * dstate).  prevBx_final is U_{T-1} (summed over ranks). */
m3_status m3_mimo_chunked_fwd(const void *x, const float *dt, const float *A,
                              const float *lam, const float *theta, const void *B,
                              const void *C, const float *D, const float *W_x,
                              const float *W_y, m3_dtype dtype, const m3_bcnorm *norm,
                              const float *h0, const float *prevBx0, const float *angle0,
                              m3_dims d, void *y, float *h_final, float *prevBx_final,
                              float *angle_final, void *workspace, size_t workspace_bytes,
                              void *stream);

/* S5 -- one SISO decode step for every (batch, head) lane.  (dotLLM pull
 * request: persistent ssm_state / cum_angle and the single-token step;
 * TorchMamba README: forward == prefill + step, cache (angle, ssm, ...).)
 * In: x_t (batch, nheads, headdim) and B_t, C_t (batch, ngroups, dstate) of
 * `dtype`; dt_t, lam_t (batch, nheads), theta_t (batch, nheads, K),
 * A, D (nheads) fp32.
 * In/out: h, prevBx (batch, nheads, dstate, headdim) fp32 and angle
 * (batch, nheads, K) fp32, updated in place.
 * Out: y_t (batch, nheads, headdim) of `dtype`.  d.seqlen is ignored. */
m3_status m3_step_decode(const void *x_t, const float *dt_t, const float *A,
                         const float *lam_t, const float *theta_t, const void *B_t,
                         const void *C_t, const float *D, m3_dtype dtype,
                         const m3_bcnorm *norm, m3_dims d, float *h, float *prevBx,
                         float *angle, void *y_t, void *stream);

/* S5 for rank R -- one MIMO decode step on the full previous-input state.
 * (dotLLM pull request, "Mamba-3 MIMO streaming decode": the state is summed
 * over ranks, the angle is rank-free; TorchMamba README, "Models": rank-R
 * update on a shared (N,P) state.)
 *   X_r = W_x[r] x_t,  U_t = sum_r Bbar_r X_r^T
 *   h <- alpha h + beta prevBx + gamma U_t,  prevBx <- U_t
 *   y_t = sum_r W_y[r] (Cbar_r^T h) + D x_t
 * Arguments as m3_step_decode plus W_x, W_y (nheads, rank, headdim) fp32,
 * each NULL for all ones; B_t, C_t are (batch, ngroups, rank, dstate);
 * QkNorm/bias as in m3_bcnorm (bias (nheads, rank, dstate)).
 * 1 <= d.rank <= 8 and headdim a multiple of 4 (else M3_ERR_UNSUPPORTED). */
m3_status m3_mimo_step_decode(const void *x_t, const float *dt_t, const float *A,
                              const float *lam_t, const float *theta_t, const void *B_t,
                              const void *C_t, const float *D, const float *W_x,
                              const float *W_y, m3_dtype dtype, const m3_bcnorm *norm,
                              m3_dims d, float *h, float *prevBx, float *angle, void *y_t,
                              void *stream);

/* One decode step on the factored previous-input state, any rank (rank 1 with
 * NULL W_x, W_y is the SISO step).  Instead of prevBx (dstate x headdim per
 * lane) the caller carries the previous token's factors (TorchMamba README,
 * "Models": the cache (angle, ssm, x_prev, b_prev)):
 *   b_prev (batch, nheads, rank, dstate) fp32: the rotated (QkNorm/bias'd) B
 *          of the previous token, per rank;
 *   x_prev (batch, nheads, headdim) fp32: the previous token's x;
 * and the previous-input term sum_r b_prev[r] (W_x[r] x_prev)^T is rebuilt on
 * the fly, so a step reads and writes only h among the (N, P) states -- about
 * half the bytes of m3_step_decode.  b_prev and x_prev are updated in place
 * (to this token's rotated B and x_t); zeros start a sequence with no
 * previous token.  All other arguments, limits and errors as
 * m3_mimo_step_decode. */
m3_status m3_step_decode_factored(const void *x_t, const float *dt_t, const float *A,
                                  const float *lam_t, const float *theta_t, const void *B_t,
                                  const void *C_t, const float *D, const float *W_x,
                                  const float *W_y, m3_dtype dtype, const m3_bcnorm *norm,
                                  m3_dims d, float *h, float *b_prev, float *x_prev,
                                  float *angle, void *y_t, void *stream);

/* Gradients of the chunked scan, each fp32 with the shape of its input
 * (dx like x; dB, dC like B, C: (batch, seqlen, ngroups, [rank,] dstate);
 * dnormw_* (dstate); dbias_* (nheads, rank, dstate); dh0, dprevBx0 like
 * h0; dangle0 (batch, nheads, K)).  Any pointer may be NULL (not wanted);
 * the others are overwritten. */
typedef struct {
    float *dx, *ddt, *dA, *dlam, *dtheta, *dB, *dC, *dD, *dW_x, *dW_y;
    float *dnormw_B, *dnormw_C, *dbias_B, *dbias_C;
    float *dh0, *dprevBx0, *dangle0;
} m3_grads;

/* Backward of the chunked forward (SISO when d.rank <= 1 and W_x, W_y are
 * NULL; rank-R MIMO otherwise, with B, C carrying the rank axis).  Training
 * needs it (TorchMamba README, "Models" and "Verification"); the forward is
 * m3_siso_chunked_fwd / m3_mimo_chunked_fwd on the same arguments.
 * For the loss L = <dy, y> + <dh_final, h_final> + <dprevBx_final,
 * prevBx_final> + <dangle_final, angle_final> it writes dL/d(input) for every
 * input into `grads`.  dy (batch, seqlen, nheads, headdim) has the dtype of
 * x and is required when seqlen > 0; the three state adjoints are fp32 in
 * the shapes of the forward's final states, each NULL for zero.
 * The gradients are computed in fp32 on the FFMA pipes, recomputing the
 * forward chunk by chunk from entering states kept in the workspace; every
 * sum runs in a fixed order, so repeated calls give identical bits.
 * workspace: at least m3_workspace_bytes(M3_WS_BWD_SISO or M3_WS_BWD_MIMO,
 * d, dtype) bytes. */
m3_status m3_chunked_bwd(const void *x, const float *dt, const float *A, const float *lam,
                         const float *theta, const void *B, const void *C, const float *D,
                         const float *W_x, const float *W_y, m3_dtype dtype,
                         const m3_bcnorm *norm, const float *h0, const float *prevBx0,
                         const float *angle0, m3_dims d, const void *dy,
                         const float *dh_final, const float *dprevBx_final,
                         const float *dangle_final, const m3_grads *grads, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Size in bytes of the scratch buffer built into the library for
 * m3_siso_chunked_fwd_noalloc (32 MiB). */
#define M3_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* The SISO chunked forward for callers that cannot allocate device memory.
 * The paper has no counterpart to this entry point; it is a deployment
 * variant of m3_siso_chunked_fwd.
 *
 * Who it is for: code that may not call cudaMalloc (or any allocator) --
 * a plugin running inside a framework that owns all device memory, or a
 * host that must not allocate once it is serving -- has nowhere to take a
 * workspace from.  This entry point takes the arguments of
 * m3_siso_chunked_fwd without the workspace, and uses instead a scratch
 * buffer of M3_NOALLOC_SCRATCH_BYTES that is part of the library: a static
 * device array.  It allocates nothing and calls no allocating routine.
 *  - Set-up: each call looks up the buffer's device address on the current
 *    device (cudaGetSymbolAddress).  CUDA loads modules lazily, so the first
 *    call on a device loads the library's module there and commits the
 *    buffer's M3_NOALLOC_SCRATCH_BYTES of device memory, which stay held
 *    until the process exits.  That first call can therefore fail with
 *    M3_ERR_CUDA when the device has no memory left (for example under a
 *    framework that has already reserved it all): make it during warm-up,
 *    and before any stream capture.  Later calls only repeat the lookup,
 *    which allocates nothing and stays valid after a device reset.
 *  - Limit: sizes whose scratch need, m3_workspace_bytes(M3_WS_SISO, d,
 *    dtype), exceeds M3_NOALLOC_SCRATCH_BYTES are rejected with
 *    M3_ERR_WORKSPACE before anything is enqueued.
 *  - Sharing: every call on a device uses the same buffer, and the buffer
 *    keeps the last call's contents (nothing in it needs to start at zero).
 *    Calls that can overlap on the GPU -- on different streams, or from
 *    different host threads -- race on it; the caller must serialise them.
 * Results, errors and all other rules are those of m3_siso_chunked_fwd. */
m3_status m3_siso_chunked_fwd_noalloc(const void *x, const float *dt, const float *A,
                                      const float *lam, const float *theta, const void *B,
                                      const void *C, const float *D, m3_dtype dtype,
                                      const m3_bcnorm *norm, const float *h0,
                                      const float *prevBx0, const float *angle0, m3_dims d,
                                      void *y, float *h_final, float *prevBx_final,
                                      float *angle_final, void *stream);

/* Workspace query for the chunked forwards. */
enum { M3_WS_SISO = 0, M3_WS_MIMO = 1, M3_WS_BWD_SISO = 2, M3_WS_BWD_MIMO = 3 };
size_t m3_workspace_bytes(int which, m3_dims d, m3_dtype dtype);

/* Static description of a status code (never NULL). */
const char *m3_status_string(m3_status s);

/* Device-side error report.  The tensor-core kernels bound every internal
 * wait (about one second); a wait that runs out makes the kernel record the
 * site, stop issuing work, drain what it has in flight and return, leaving
 * its outputs undefined.  This call synchronises `stream`, returns
 * M3_ERR_TIMEOUT if any kernel recorded such an error since the last call
 * (and clears it), M3_ERR_CUDA if the stream reports a CUDA error, else
 * M3_OK.  When `site` is not NULL it receives the recorded wait site (0 when
 * none).  It is the one entry point that synchronises. */
m3_status m3_device_error(void *stream, int *site);

/* Self-test of the timeout path.  Enqueues one kernel that waits, with the
 * library's bounded wait, on a barrier that nothing ever completes: after
 * about one second the wait gives up and records M3_SELFTEST_SITE in the
 * device error word, and the kernel returns normally (no fault, no trap; the
 * context stays usable).  m3_device_error then reports M3_ERR_TIMEOUT with
 * that site.  Returns M3_OK once enqueued. */
#define M3_SELFTEST_SITE 99
m3_status m3_selftest_bounded_wait(void *stream);

/* Host-side failure injection, for testing callers' error paths.  After
 * this call the next n entry-point calls that pass their argument checks
 * return M3_ERR_CUDA, as a failed launch would, and enqueue nothing (their
 * outputs are left as they were).  n <= 0 turns it off.  Calls that fail
 * their checks still return their own status and do not count.  Nothing on
 * the device is touched, so it is safe with or without a GPU. */
void m3_debug_fail_next_launches(int n);

/* Number of kernels the library has enqueued since it was loaded (host-side
 * counter, incremented once per launch; used to count launches in a timed
 * region). */
uint64_t m3_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* M3_H */
