// k_decode.cu -- one SISO decode step for every (b, h) lane (memory-bound).
//
// (dotLLM pull request: persistent ssm_state and cum_angle threaded through
// single-token steps; TorchMamba README: forward == prefill + step.)
//   Phi <- Phi + dt theta;  Bbar, Cbar = R(Phi) (QkNorm/bias'd) B, C
//   U = Bbar x^T;  h <- alpha h + beta prev_Bx + gamma U;  prev_Bx <- U
//   y = Cbar^T h + D x
// The state (h and prev_Bx, 2 x N x P fp32 per lane, read and written) is all
// the traffic that matters; every thread streams VEC-wide rows of it.  Head h
// reads the B/C row of group h / (H / G); pairs j >= K do not rotate.
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
__global__ void __launch_bounds__(256, 5) k_decode(DecodeArgs a) {
    using V = typename vecf<VEC>::type;
    const int64_t lane = blockIdx.x, h = lane % a.H;
    const int P = (int)a.P, N = (int)a.N, NP2 = N / 2, K = (int)a.K;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int64_t row = (lane / a.H) * a.G + h / (a.H / a.G);   // the group's B/C row
    const T *x = static_cast<const T *>(a.x);
    const T *Bg = static_cast<const T *>(a.B) + row * N;
    const T *Cg = static_cast<const T *>(a.C) + row * N;
    T *y = static_cast<T *>(a.y);

    extern __shared__ float sm[];
    float *Bb = sm;            // N
    float *Cb = Bb + N;        // N
    float *red = Cb + N;       // 32
    float *ypart = red + 32;   // ngroups * P

    const int PV = P / VEC;              // vectors per state row
    const int ngroups = nt / PV;         // rows streamed concurrently
    const int pv = tid % PV, ng = tid / PV;
    {   // start pulling my rows of h and prev_Bx into L2 now, so the state
        // stream below finds them there instead of waiting on HBM after the prologue
        const V *hq = reinterpret_cast<const V *>(a.h + lane * (int64_t)N * P) + pv;
        const V *uq = reinterpret_cast<const V *>(a.prevBx + lane * (int64_t)N * P) + pv;
        if (ng < ngroups)
            for (int n = ng; n < N; n += ngroups) {
                asm volatile("prefetch.global.L2 [%0];" ::"l"(hq + n * PV));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(uq + n * PV));
            }
    }

    const float dl = a.dt[lane], lm = a.lam[lane];
    const float al = expf(dl * a.A[h]);
    const float be = (1.f - lm) * dl * al;
    const float ga = lm * dl;

    float invB = 1.f, invC = 1.f;
    if (a.nrm.wB || a.nrm.wC) {
        float sb = 0.f, sc = 0.f;
        for (int n = tid; n < N; n += nt) {
            const float vb = ldf(Bg, n), vc = ldf(Cg, n);
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
        float sn = 0.f, cn = 1.f;
        if (j < K) {
            const float phi = a.angle[lane * K + j] + dl * a.theta[lane * K + j];
            a.angle[lane * K + j] = phi;
            sincosf(phi, &sn, &cn);
        }
        float b0 = ldf(Bg, 2 * j), b1 = ldf(Bg, 2 * j + 1);
        float c0 = ldf(Cg, 2 * j), c1 = ldf(Cg, 2 * j + 1);
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

// ---------------------------------------------------------------------------
// Rank-R decode step, on the full previous-input state (prev_Bx, N x P per
// lane) or on its factors (dotLLM pull request, "Mamba-3 MIMO streaming
// decode": the state is summed over ranks and the angle is rank-free;
// TorchMamba README, "Models": the cache (angle, ssm, x_prev, b_prev)):
//   X_r = W_x[r] x_t,  U_t = sum_r Bbar_r X_r^T
//   U_prev = prev_Bx  or  sum_r b_prev[r] (W_x[r] x_prev)^T   (factored)
//   h <- alpha h + beta U_prev + gamma U_t
//   y = sum_r W_y[r] (Cbar_r^T h) + D x_t
//   prev_Bx <- U_t   or   b_prev <- Bbar, x_prev <- x_t      (factored)
// One CTA per (b, h) lane; rank bound RT (R <= RT, the rest predicated off);
// threads stream 4-wide rows of h (and prev_Bx).  The factored form reads and
// writes only h, so a step moves about half the bytes of the full form.
// ---------------------------------------------------------------------------
template <typename T, int RT, bool FACT>
__global__ void __launch_bounds__(256) k_decode_gen(DecodeArgs a) {
    constexpr int VEC = 4;
    const int64_t lane = blockIdx.x, h = lane % a.H;
    const int P = (int)a.P, N = (int)a.N, NP2 = N / 2, R = (int)a.R, K = (int)a.K;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int64_t grow = (lane / a.H) * a.G + h / (a.H / a.G);  // the group's B/C rows
    const T *x = static_cast<const T *>(a.x);
    const T *Bg = static_cast<const T *>(a.B) + grow * R * N;
    const T *Cg = static_cast<const T *>(a.C) + grow * R * N;
    T *y = static_cast<T *>(a.y);

    extern __shared__ float sm[];
    float *Bb = sm;                 // RT x N  rotated B of this token
    float *Cb = Bb + RT * N;        // RT x N  rotated C
    float *Pb = Cb + RT * N;        // RT x N  b_prev (factored form)
    float *red = Pb + RT * N;       // 32
    float *phs = red + 32;          // N/2 angles of this token
    float *ypart = phs + N / 2;     // ngroups x RT x P

    const int PV = P / VEC;              // vectors per state row
    const int ngroups = nt / PV;         // rows streamed concurrently
    const int pv = tid % PV, ng = tid / PV;
    float4 *hp = reinterpret_cast<float4 *>(a.h + lane * (int64_t)N * P);
    // start pulling my rows of h into L2 now: the state stream below then
    // finds them there instead of waiting on HBM after the prologue
    if (ng < ngroups)
        for (int n = ng; n < N; n += ngroups)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(hp + n * PV + pv));

    const float dl = a.dt[lane], lm = a.lam[lane];
    const float al = expf(dl * a.A[h]);
    const float be = (1.f - lm) * dl * al;
    const float ga = lm * dl;

    // QkNorm inverse RMS per rank
    float invB[RT], invC[RT];
#pragma unroll
    for (int r = 0; r < RT; r++) { invB[r] = 1.f; invC[r] = 1.f; }
    if (a.nrm.wB || a.nrm.wC) {
#pragma unroll
        for (int r = 0; r < RT; r++) {
            if (r >= R) break;
            float sb = 0.f, sc = 0.f;
            for (int n = tid; n < N; n += nt) {
                const float vb = ldf(Bg, r * N + n), vc = ldf(Cg, r * N + n);
                sb += vb * vb;
                sc += vc * vc;
            }
            sb = block_sum(sb, red);
            __syncthreads();
            sc = block_sum(sc, red);
            __syncthreads();
            invB[r] = rsqrtf(sb / N + a.nrm.eps);
            invC[r] = rsqrtf(sc / N + a.nrm.eps);
        }
    }
    if (FACT)
        for (int k = tid; k < R * N; k += nt) Pb[k] = a.bprev[lane * R * N + k];
    for (int j = tid; j < K; j += nt) {
        const float phi = a.angle[lane * K + j] + dl * a.theta[lane * K + j];
        a.angle[lane * K + j] = phi;
        phs[j] = phi;
    }
    __syncthreads();
    // one (pair, rank) per thread: every rank's loads in flight at once
    for (int it = tid; it < R * NP2; it += nt) {
        const int j = it % NP2, r = it / NP2;
        float sn = 0.f, cn = 1.f;
        if (j < K) sincosf(phs[j], &sn, &cn);
        {
            const int64_t o = r * N + 2 * j;
            float b0 = ldf(Bg, o), b1 = ldf(Bg, o + 1), c0 = ldf(Cg, o), c1 = ldf(Cg, o + 1);
            float ib = 1.f, ic = 1.f;   // this rank's inverse RMS (selected, not indexed)
#pragma unroll
            for (int rr = 0; rr < RT; rr++)
                if (rr == r) { ib = invB[rr]; ic = invC[rr]; }
            if (a.nrm.wB) { b0 *= ib * a.nrm.wB[2 * j]; b1 *= ib * a.nrm.wB[2 * j + 1]; }
            if (a.nrm.wC) { c0 *= ic * a.nrm.wC[2 * j]; c1 *= ic * a.nrm.wC[2 * j + 1]; }
            const int64_t bo = (h * R + r) * N + 2 * j;
            if (a.nrm.biasB) { b0 += a.nrm.biasB[bo]; b1 += a.nrm.biasB[bo + 1]; }
            if (a.nrm.biasC) { c0 += a.nrm.biasC[bo]; c1 += a.nrm.biasC[bo + 1]; }
            Bb[r * N + 2 * j] = cn * b0 - sn * b1;
            Bb[r * N + 2 * j + 1] = sn * b0 + cn * b1;
            Cb[r * N + 2 * j] = cn * c0 - sn * c1;
            Cb[r * N + 2 * j + 1] = sn * c0 + cn * c1;
        }
    }
    __syncthreads();

    // Small ranks keep X_r = W_x[r] x (and W_x[r] x_prev) per rank; ranks 4
    // and 8 keep W_x[r] alone and scale the rank sums by x (x_prev) after, which
    // holds half the registers:  U_t[n][p] = x[p] sum_r Bbar_r[n] W_x[r][p].
    constexpr bool WF = RT >= 4;
    constexpr int RX = WF ? 1 : RT;                 // per-rank products kept
    float xv[VEC], xq[VEC], W[RT][VEC], X[RX][VEC], Xp[RX][VEC], Y[RT][VEC];
#pragma unroll
    for (int k = 0; k < VEC; k++) {
        xv[k] = ldf(x, lane * P + pv * VEC + k);
        xq[k] = FACT ? a.xprev[lane * P + pv * VEC + k] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < RT; r++) {
#pragma unroll
        for (int k = 0; k < VEC; k++) {
            const int p = pv * VEC + k;
            W[r][k] = r < R ? (a.Wx ? a.Wx[(h * R + r) * P + p] : 1.f) : 0.f;
            Y[r][k] = 0.f;
            if (!WF) {
                X[r < RX ? r : 0][k] = W[r][k] * xv[k];
                Xp[r < RX ? r : 0][k] = W[r][k] * xq[k];
            }
        }
    }
    if (ng < ngroups) {
        float4 *up = FACT ? nullptr : reinterpret_cast<float4 *>(a.prevBx + lane * (int64_t)N * P);
#pragma unroll 2
        for (int n = ng; n < N; n += ngroups) {
            const float4 hq = hp[n * PV + pv];
            float hv[VEC] = {hq.x, hq.y, hq.z, hq.w}, uv[VEC], ut[VEC];
            if (!FACT) {
                const float4 uq = up[n * PV + pv];
                uv[0] = uq.x; uv[1] = uq.y; uv[2] = uq.z; uv[3] = uq.w;
            }
#pragma unroll
            for (int k = 0; k < VEC; k++) {
                ut[k] = 0.f;
                if (FACT) uv[k] = 0.f;
            }
#pragma unroll
            for (int r = 0; r < RT; r++) {
                const float bn = Bb[r * N + n], pn = FACT ? Pb[r * N + n] : 0.f;
#pragma unroll
                for (int k = 0; k < VEC; k++) {
                    ut[k] = fmaf(bn, WF ? W[r][k] : X[r < RX ? r : 0][k], ut[k]);
                    if (FACT) uv[k] = fmaf(pn, WF ? W[r][k] : Xp[r < RX ? r : 0][k], uv[k]);
                }
            }
            if (WF) {
#pragma unroll
                for (int k = 0; k < VEC; k++) {
                    ut[k] *= xv[k];
                    if (FACT) uv[k] *= xq[k];
                }
            }
#pragma unroll
            for (int k = 0; k < VEC; k++) hv[k] = al * hv[k] + be * uv[k] + ga * ut[k];
#pragma unroll
            for (int r = 0; r < RT; r++) {
                const float cn = Cb[r * N + n];
#pragma unroll
                for (int k = 0; k < VEC; k++) Y[r][k] = fmaf(cn, hv[k], Y[r][k]);
            }
            hp[n * PV + pv] = make_float4(hv[0], hv[1], hv[2], hv[3]);
            if (!FACT) up[n * PV + pv] = make_float4(ut[0], ut[1], ut[2], ut[3]);
        }
#pragma unroll
        for (int r = 0; r < RT; r++)
#pragma unroll
            for (int k = 0; k < VEC; k++) ypart[(ng * RT + r) * P + pv * VEC + k] = Y[r][k];
    }
    __syncthreads();
    for (int p = tid; p < P; p += nt) {
        float s = 0.f;
        for (int r = 0; r < R; r++) {
            float yr = 0.f;
            for (int g = 0; g < ngroups; g++) yr += ypart[(g * RT + r) * P + p];
            s += (a.Wy ? a.Wy[(h * R + r) * P + p] : 1.f) * yr;
        }
        const float xp_new = ldf(x, lane * P + p);
        stf(y, lane * P + p, s + a.D[h] * xp_new);
        if (FACT) a.xprev[lane * P + p] = xp_new;
    }
    if (FACT)
        for (int k = tid; k < R * N; k += nt) a.bprev[lane * R * N + k] = Bb[k];
}

template <typename T, int RT>
static cudaError_t launch_decode_gen_rt(const DecodeArgs &a, bool factored, cudaStream_t s) {
    const int threads = 256;
    const int ngroups = threads / (int)(a.P / 4);
    const size_t smem = sizeof(float) * (3 * RT * a.N + 32 + a.N / 2 + (size_t)ngroups * RT * a.P);
    // rank 8 at dstate 256 needs about 57 KB, past the 48 KB a launch gets by default
    if (factored) {
        cudaFuncSetAttribute(k_decode_gen<T, RT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_decode_gen<T, RT, true><<<(unsigned)(a.Bt * a.H), threads, smem, s>>>(a);
    } else {
        cudaFuncSetAttribute(k_decode_gen<T, RT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_decode_gen<T, RT, false><<<(unsigned)(a.Bt * a.H), threads, smem, s>>>(a);
    }
    count_launch();
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_decode_gen_t(const DecodeArgs &a, bool factored, cudaStream_t s) {
    if (a.R <= 1) return launch_decode_gen_rt<T, 1>(a, factored, s);
    if (a.R <= 2) return launch_decode_gen_rt<T, 2>(a, factored, s);
    if (a.R <= 4) return launch_decode_gen_rt<T, 4>(a, factored, s);
    return launch_decode_gen_rt<T, 8>(a, factored, s);
}

cudaError_t launch_decode_gen(const DecodeArgs &a, m3_dtype dt, bool factored, cudaStream_t s) {
    if (a.Bt * a.H == 0) return cudaSuccess;
    return dt == M3_BF16 ? launch_decode_gen_t<__nv_bfloat16>(a, factored, s)
                         : launch_decode_gen_t<float>(a, factored, s);
}

}  // namespace m3
