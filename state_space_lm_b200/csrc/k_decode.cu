// k_decode.cu -- one SISO decode step for every (b, h) lane (memory-bound).
//
// (dotLLM pull request: persistent ssm_state and cum_angle threaded through
// single-token steps; TorchMamba README: forward == prefill + step.)
//   Phi <- Phi + dt theta;  Bbar, Cbar = R(Phi) (QkNorm/bias'd) B, C
//   U = Bbar x^T;  h <- alpha h + beta prev_Bx + gamma U;  prev_Bx <- U
//   y = Cbar^T h + D x
// The state (h and prev_Bx, 2 x N x P fp32 per lane, read and written) is all
// the traffic that matters; every thread streams VEC-wide rows of it.
#include "m3_internal.cuh"

namespace m3 {

template <int VEC> struct vecf;
template <> struct vecf<4> {
    using type = float4;
    static __device__ __forceinline__ void unpack(const float4 &v, float *o) {
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
    static __device__ __forceinline__ float4 pack(const float *o) { return make_float4(o[0], o[1], o[2], o[3]); }
};
template <> struct vecf<1> {
    using type = float;
    static __device__ __forceinline__ void unpack(const float &v, float *o) { o[0] = v; }
    static __device__ __forceinline__ float pack(const float *o) { return o[0]; }
};

template <typename T, int VEC>
__global__ void __launch_bounds__(256) k_decode(DecodeArgs a) {
    using V = typename vecf<VEC>::type;
    const int64_t lane = blockIdx.x, h = lane % a.H;
    const int P = (int)a.P, N = (int)a.N, NP2 = N / 2;
    const int tid = threadIdx.x, nt = blockDim.x;
    const T *x = static_cast<const T *>(a.x);
    const T *Bg = static_cast<const T *>(a.B);
    const T *Cg = static_cast<const T *>(a.C);
    T *y = static_cast<T *>(a.y);

    extern __shared__ float sm[];
    float *Bb = sm;            // N
    float *Cb = Bb + N;        // N
    float *red = Cb + N;       // 32
    float *ypart = red + 32;   // ngroups * P

    const float dl = a.dt[lane], lm = a.lam[lane];
    const float al = expf(dl * a.A[h]);
    const float be = (1.f - lm) * dl * al;
    const float ga = lm * dl;

    float invB = 1.f, invC = 1.f;
    if (a.nrm.wB || a.nrm.wC) {
        float sb = 0.f, sc = 0.f;
        for (int n = tid; n < N; n += nt) {
            const float vb = ldf(Bg, lane * N + n), vc = ldf(Cg, lane * N + n);
            sb += vb * vb;
            sc += vc * vc;
        }
        sb = block_sum(sb, red);
        __syncthreads();
        sc = block_sum(sc, red);
        invB = rsqrtf(sb / N + a.nrm.eps);
        invC = rsqrtf(sc / N + a.nrm.eps);
    }
    for (int j = tid; j < NP2; j += nt) {
        const float phi = a.angle[lane * NP2 + j] + dl * a.theta[lane * NP2 + j];
        a.angle[lane * NP2 + j] = phi;
        float sn, cn;
        sincosf(phi, &sn, &cn);
        float b0 = ldf(Bg, lane * N + 2 * j), b1 = ldf(Bg, lane * N + 2 * j + 1);
        float c0 = ldf(Cg, lane * N + 2 * j), c1 = ldf(Cg, lane * N + 2 * j + 1);
        if (a.nrm.wB) { b0 *= invB * a.nrm.wB[2 * j]; b1 *= invB * a.nrm.wB[2 * j + 1]; }
        if (a.nrm.wC) { c0 *= invC * a.nrm.wC[2 * j]; c1 *= invC * a.nrm.wC[2 * j + 1]; }
        if (a.nrm.biasB) { b0 += a.nrm.biasB[h * N + 2 * j]; b1 += a.nrm.biasB[h * N + 2 * j + 1]; }
        if (a.nrm.biasC) { c0 += a.nrm.biasC[h * N + 2 * j]; c1 += a.nrm.biasC[h * N + 2 * j + 1]; }
        Bb[2 * j] = cn * b0 - sn * b1;
        Bb[2 * j + 1] = sn * b0 + cn * b1;
        Cb[2 * j] = cn * c0 - sn * c1;
        Cb[2 * j + 1] = sn * c0 + cn * c1;
    }
    __syncthreads();

    const int PV = P / VEC;              // vectors per state row
    const int ngroups = nt / PV;         // rows streamed concurrently
    const int pv = tid % PV, ng = tid / PV;
    float xv[VEC], yacc[VEC];
#pragma unroll
    for (int k = 0; k < VEC; k++) {
        xv[k] = ldf(x, lane * P + pv * VEC + k);
        yacc[k] = 0.f;
    }
    if (ng < ngroups) {
        V *hp = reinterpret_cast<V *>(a.h + lane * (int64_t)N * P);
        V *up = reinterpret_cast<V *>(a.prevBx + lane * (int64_t)N * P);
#pragma unroll 4
        for (int n = ng; n < N; n += ngroups) {
            float hv[VEC], uv[VEC];
            vecf<VEC>::unpack(hp[n * PV + pv], hv);
            vecf<VEC>::unpack(up[n * PV + pv], uv);
            const float bn = Bb[n], cn = Cb[n];
#pragma unroll
            for (int k = 0; k < VEC; k++) {
                const float u = bn * xv[k];
                const float hn = al * hv[k] + be * uv[k] + ga * u;
                yacc[k] += cn * hn;
                hv[k] = hn;
                uv[k] = u;
            }
            hp[n * PV + pv] = vecf<VEC>::pack(hv);
            up[n * PV + pv] = vecf<VEC>::pack(uv);
        }
#pragma unroll
        for (int k = 0; k < VEC; k++) ypart[ng * P + pv * VEC + k] = yacc[k];
    }
    __syncthreads();
    for (int p = tid; p < P; p += nt) {
        float s = 0.f;
        for (int k = 0; k < ngroups; k++) s += ypart[k * P + p];
        stf(y, lane * P + p, s + a.D[h] * ldf(x, lane * P + p));
    }
}

template <typename T>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t s) {
    const int64_t lanes = a.Bt * a.H;
    const int threads = 256;
    if (a.P % 4 == 0) {
        const int ngroups = threads / (int)(a.P / 4);
        const size_t smem = sizeof(float) * (2 * a.N + 32 + (size_t)ngroups * a.P);
        k_decode<T, 4><<<(unsigned)lanes, threads, smem, s>>>(a);
    } else {
        const int ngroups = threads / (int)a.P;
        const size_t smem = sizeof(float) * (2 * a.N + 32 + (size_t)ngroups * a.P);
        k_decode<T, 1><<<(unsigned)lanes, threads, smem, s>>>(a);
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, m3_dtype dt, cudaStream_t s) {
    if (a.Bt * a.H == 0) return cudaSuccess;
    return dt == M3_BF16 ? launch_decode_t<__nv_bfloat16>(a, s) : launch_decode_t<float>(a, s);
}

}  // namespace m3
