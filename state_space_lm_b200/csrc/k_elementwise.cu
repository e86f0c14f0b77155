// k_elementwise.cu -- S1 (trapezoidal discretization) and S2 (QkNorm +
// BC-bias + data-dependent RoPE) as standalone bandwidth-bound kernels.
//
// Discretization (dotLLM pull request, "Stage A: Mamba3Discretize"; TorchMamba
// README, "Math notes", Prop. 1): alpha = exp(dt A), beta = (1-lam) dt alpha,
// gamma = lam dt.
// Rotation (dotLLM pull request, "Stage A: Mamba3DataRoPE"; TorchMamba README,
// "Math notes", Props. 2-4): Phi_t = Phi_{t-1} + dt_t theta_t per pair, each
// adjacent pair (2i, 2i+1) of B and C rotated by +Phi_t.
#include "m3_internal.cuh"

namespace m3 {

__global__ void __launch_bounds__(256) k_discretize(const float *__restrict__ dt,
                                                   const float *__restrict__ A,
                                                   const float *__restrict__ lam, int64_t n,
                                                   int64_t H, float *__restrict__ al,
                                                   float *__restrict__ be,
                                                   float *__restrict__ ga) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t n4 = n >> 2;
    // four elements per thread-iteration: 16-byte loads and stores
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n4; v += stride) {
        const float4 d = reinterpret_cast<const float4 *>(dt)[v];
        const float4 l = reinterpret_cast<const float4 *>(lam)[v];
        const int64_t i = v << 2;
        float dd[4] = {d.x, d.y, d.z, d.w}, ll[4] = {l.x, l.y, l.z, l.w};
        float oa[4], ob[4], og[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float a = expf(dd[k] * A[(i + k) % H]);
            oa[k] = a;
            ob[k] = (1.f - ll[k]) * dd[k] * a;
            og[k] = ll[k] * dd[k];
        }
        reinterpret_cast<float4 *>(al)[v] = make_float4(oa[0], oa[1], oa[2], oa[3]);
        reinterpret_cast<float4 *>(be)[v] = make_float4(ob[0], ob[1], ob[2], ob[3]);
        reinterpret_cast<float4 *>(ga)[v] = make_float4(og[0], og[1], og[2], og[3]);
    }
    for (int64_t i = (n4 << 2) + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float a = expf(dt[i] * A[i % H]);
        al[i] = a;
        be[i] = (1.f - lam[i]) * dt[i] * a;
        ga[i] = lam[i] * dt[i];
    }
}

cudaError_t launch_discretize(const float *dt, const float *A, const float *lam, int64_t Bt,
                              int64_t T, int64_t H, float *al, float *be, float *ga,
                              cudaStream_t s) {
    const int64_t n = Bt * T * H;
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n / 4 + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_discretize<<<(unsigned)blocks, 256, 0, s>>>(dt, A, lam, n, H, al, be, ga);
    count_launch();
    return cudaGetLastError();
}

// ---- pair access ----------------------------------------------------------
__device__ __forceinline__ float2 ld2(const float *p, int64_t i) {
    return *reinterpret_cast<const float2 *>(p + i);
}
__device__ __forceinline__ float2 ld2(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p + i));
}
__device__ __forceinline__ void st2(float *p, int64_t i, float a, float b) {
    *reinterpret_cast<float2 *>(p + i) = make_float2(a, b);
}
__device__ __forceinline__ void st2(__nv_bfloat16 *p, int64_t i, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p + i) = __floats2bfloat162_rn(a, b);
}

// One CTA per (b, h) lane walks the sequence in tiles of ny*SEG tokens.  The
// thread grid is (ny rows) x (N/2 pairs): in pass 1 every row sums dt*theta
// over its SEG tokens, the rows' partial sums give each row its starting
// angle, and pass 2 walks the same tokens again rotating B and C.  Only pairs
// j < K turn (partial RoPE); the rest are copied with QkNorm/bias applied.
// The lane reads the B/C rows of its group h / (H / G) and writes per head.
template <typename T>
__global__ void __launch_bounds__(256) k_rope(RopeArgs a) {
    constexpr int SEG = 16;
    const int64_t lane = blockIdx.x, b = lane / a.H, h = lane % a.H;
    const int64_t Tn = a.T, H = a.H, G = a.G, hg = h / (H / G);
    const int N = (int)a.N, R = (int)a.R, NP2 = N / 2, K = (int)a.K;
    const int ny = min((int)blockDim.x / NP2, 64);
    const int ty = threadIdx.x / NP2, j = threadIdx.x % NP2;
    const bool active = ty < ny;
    const int TT = ny * SEG;
    const T *B = static_cast<const T *>(a.B);
    const T *C = static_cast<const T *>(a.C);
    T *Bo = static_cast<T *>(a.Bo);
    T *Co = static_cast<T *>(a.Co);
    const bool has_norm = a.nrm.wB || a.nrm.wC;

    extern __shared__ float sm[];
    float *part = sm;                 // ny * NP2
    float *carry = part + ny * NP2;   // NP2
    float *invB = carry + NP2;        // TT * R
    float *invC = invB + TT * R;      // TT * R

    for (int k = threadIdx.x; k < NP2; k += blockDim.x)
        carry[k] = (a.angle0 && k < K) ? a.angle0[lane * K + k] : 0.f;
    __syncthreads();

    const int warp = threadIdx.x >> 5, l32 = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int64_t t0 = 0; t0 < Tn; t0 += TT) {
        float s = 0.f;
        if (active) {
            for (int k = 0; k < SEG && j < K; k++) {
                const int64_t t = t0 + ty * SEG + k;
                if (t < Tn) {
                    const int64_t bt = (b * Tn + t) * H + h;
                    s += a.dt[bt] * a.theta[bt * K + j];
                }
            }
            part[ty * NP2 + j] = s;
        }
        if (has_norm) {
            for (int row = warp; row < TT * R; row += nw) {
                const int64_t t = t0 + row / R;
                if (t >= Tn) continue;
                const int64_t base = (((b * Tn + t) * G + hg) * R + row % R) * N;
                float sb = 0.f, sc = 0.f;
                for (int n = l32; n < N; n += 32) {
                    const float vb = ldf(B, base + n), vc = ldf(C, base + n);
                    sb += vb * vb;
                    sc += vc * vc;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    sb += __shfl_xor_sync(0xffffffffu, sb, o);
                    sc += __shfl_xor_sync(0xffffffffu, sc, o);
                }
                if (l32 == 0) {
                    invB[row] = rsqrtf(sb / N + a.nrm.eps);
                    invC[row] = rsqrtf(sc / N + a.nrm.eps);
                }
            }
        }
        __syncthreads();
        float phi = 0.f, tot = 0.f;
        if (active) {
            phi = carry[j];
            tot = carry[j];
            for (int k = 0; k < ny; k++) {
                const float v = part[k * NP2 + j];
                if (k < ty) phi += v;
                tot += v;
            }
        }
        __syncthreads();
        if (active && ty == 0) carry[j] = tot;
        if (active) {
            for (int k = 0; k < SEG; k++) {
                const int tl = ty * SEG + k;
                const int64_t t = t0 + tl;
                if (t >= Tn) break;
                const int64_t bt = (b * Tn + t) * H + h;
                float sn = 0.f, cs = 1.f;
                if (j < K) {
                    phi += a.dt[bt] * a.theta[bt * K + j];
                    sincosf(phi, &sn, &cs);
                }
                for (int r = 0; r < R; r++) {
                    const int64_t idx = (bt * R + r) * N + 2 * j;
                    const int64_t src = (((b * Tn + t) * G + hg) * R + r) * N + 2 * j;
                    float2 bv = ld2(B, src), cv = ld2(C, src);
                    if (a.nrm.wB) {
                        const float iv = invB[tl * R + r];
                        bv.x *= iv * a.nrm.wB[2 * j];
                        bv.y *= iv * a.nrm.wB[2 * j + 1];
                    }
                    if (a.nrm.wC) {
                        const float iv = invC[tl * R + r];
                        cv.x *= iv * a.nrm.wC[2 * j];
                        cv.y *= iv * a.nrm.wC[2 * j + 1];
                    }
                    if (a.nrm.biasB) {
                        bv.x += a.nrm.biasB[(h * R + r) * N + 2 * j];
                        bv.y += a.nrm.biasB[(h * R + r) * N + 2 * j + 1];
                    }
                    if (a.nrm.biasC) {
                        cv.x += a.nrm.biasC[(h * R + r) * N + 2 * j];
                        cv.y += a.nrm.biasC[(h * R + r) * N + 2 * j + 1];
                    }
                    if (j < K) {
                        st2(Bo, idx, cs * bv.x - sn * bv.y, sn * bv.x + cs * bv.y);
                        st2(Co, idx, cs * cv.x - sn * cv.y, sn * cv.x + cs * cv.y);
                    } else {
                        st2(Bo, idx, bv.x, bv.y);
                        st2(Co, idx, cv.x, cv.y);
                    }
                }
                if (t == Tn - 1 && a.angle_out && j < K) a.angle_out[lane * K + j] = phi;
            }
        }
        __syncthreads();
    }
    if (Tn == 0 && a.angle_out)
        for (int k = threadIdx.x; k < K; k += blockDim.x) a.angle_out[lane * K + k] = carry[k];
}

cudaError_t launch_rope(const RopeArgs &a, m3_dtype dt, cudaStream_t s) {
    const int64_t lanes = a.Bt * a.H;
    if (lanes == 0) return cudaSuccess;
    const int NP2 = (int)(a.N / 2);
    const int threads = 256;
    const int ny = threads / NP2 < 64 ? threads / NP2 : 64;
    const int TT = ny * 16;
    const size_t smem = sizeof(float) * ((size_t)ny * NP2 + NP2 + 2 * (size_t)TT * a.R);
    if (dt == M3_BF16) {
        cudaFuncSetAttribute(k_rope<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_rope<__nv_bfloat16><<<(unsigned)lanes, threads, smem, s>>>(a);
    } else {
        cudaFuncSetAttribute(k_rope<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_rope<float><<<(unsigned)lanes, threads, smem, s>>>(a);
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace m3
