// m3_internal.cuh -- shared declarations of the CUDA side (not part of the ABI).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "m3.h"

namespace m3 {

// ---- element access: every kernel computes in fp32 ------------------------
__device__ __forceinline__ float ldf(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void stf(float *p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }

// Sum over the whole block (blockDim.x a multiple of 32, <= 1024).  `red`
// holds 32 floats of shared memory.  Every thread receives the total.
__device__ __forceinline__ float block_sum(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < nw; i++) s += red[i];
    return s;
}

// ---- launch descriptions (host fills, kernels read) ----------------------
struct NormArgs {
    const float *wB, *wC, *biasB, *biasC;
    float eps;
};

struct ScanArgs {
    const void *x, *B, *C;
    const float *dt, *A, *lam, *theta, *D, *Wx, *Wy;
    const float *h0, *prevBx0, *angle0;
    NormArgs nrm;
    void *y;
    float *h_out, *prevBx_out, *angle_out;
    int64_t Bt, T, H, P, N, R;
    int64_t G = 0, K = 0;  // B/C groups (H % G == 0) and rotated pairs (K <= N/2), resolved
    int Q;             // chunk length actually used by the kernel
    int mimo_layout;   // B/C carry a rank axis
    void *ws;          // caller's workspace (may be null when none is needed)
};

struct DecodeArgs {
    const void *x, *B, *C;
    const float *dt, *A, *lam, *theta, *D;
    NormArgs nrm;
    float *h, *prevBx, *angle;
    void *y;
    int64_t Bt, H, P, N;
    int64_t G = 0, K = 0;  // B/C groups and rotated pairs, resolved
    // rank-R and factored-state decode (k_decode_gen)
    const float *Wx = nullptr, *Wy = nullptr;   // (H, R, P), NULL = ones
    float *bprev = nullptr, *xprev = nullptr;   // factored previous-input state
    int64_t R = 1;
};

struct RopeArgs {
    const void *B, *C;
    const float *theta, *dt, *angle0;
    NormArgs nrm;
    void *Bo, *Co;
    float *angle_out;
    int64_t Bt, T, H, R, N;
    int64_t G = 0, K = 0;  // B/C groups and rotated pairs, resolved
};

struct BwdArgs {
    const void *x, *B, *C, *dy;
    const float *dt, *A, *lam, *theta, *D, *Wx, *Wy;
    const float *h0, *prevBx0, *angle0;
    const float *dh, *du, *da;     // adjoints of h_final, prevBx_final, angle_final (NULL = 0)
    NormArgs nrm;
    // gradients (each NULL = not wanted), fp32
    float *dx, *ddt, *dA, *dlam, *dtheta, *dB, *dC, *dD, *dWx, *dWy, *dwB, *dwC, *dbB, *dbC, *dh0, *du0, *da0;
    int64_t Bt, T, H, P, N, R, G, K;
    int Q;                          // chunk length used by the backward kernels
    float *ws;                      // caller's workspace
    size_t ws_slots = 0, ws_partial = 0, ws_dBh = 0, ws_dCh = 0;   // offsets (floats), set by the launcher
};

// Host launchers (each returns cudaSuccess or the launch error).
cudaError_t launch_discretize(const float *dt, const float *A, const float *lam, int64_t Bt,
                              int64_t T, int64_t H, float *al, float *be, float *ga,
                              cudaStream_t s);
cudaError_t launch_rope(const RopeArgs &a, m3_dtype dt, cudaStream_t s);
cudaError_t launch_scan_simt(const ScanArgs &a, m3_dtype dt, cudaStream_t s);
size_t scan_simt_smem_bytes(int64_t P, int64_t N, int64_t R, int Q);
int scan_simt_chunk(int64_t P, int64_t N, int64_t R, int64_t chunk);
cudaError_t launch_decode(const DecodeArgs &a, m3_dtype dt, cudaStream_t s);
// rank R (1..8), full (prevBx) or factored (bprev, xprev) previous-input state; headdim % 4 == 0
cudaError_t launch_decode_gen(const DecodeArgs &a, m3_dtype dt, bool factored, cudaStream_t s);
// tensor-core SISO scan (bf16, headdim 64, dState 128, chunk 64)
bool scan_tc_supported(const ScanArgs &a, m3_dtype dt);
cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t s);
int scan_tc_error_and_clear(cudaStream_t s);
// one bounded wait on a barrier nothing completes (tests the timeout path)
cudaError_t launch_wait_selftest(int site, cudaStream_t s);
size_t scan_tc_workspace_bytes(int64_t Bt, int64_t H, int64_t T);

// backward of the chunked scan (FFMA): chunk length that fits, workspace, launch
int bwd_chunk(int64_t P, int64_t N, int64_t R, int64_t K, int64_t chunk);
size_t scan_bwd_workspace_bytes(const BwdArgs &a);
cudaError_t launch_scan_bwd(const BwdArgs &a, m3_dtype dt, cudaStream_t s);

// Launch counter shared by all launchers.
void count_launch(int n = 1);

}  // namespace m3
