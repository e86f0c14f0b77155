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
template <> struct vecf<2> {
    using type = float2;
    static __device__ __forceinline__ void unpack(const float2 &v, float *o) { o[0] = v.x; o[1] = v.y; }
    static __device__ __forceinline__ float2 pack(const float *o) { return make_float2(o[0], o[1]); }
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
// One CTA per (b, h) lane; rank bound RT (R <= RT, the ranks past R are zero
// rows).  The factored form reads and writes only h, so a step moves about
// half the bytes of the full form.  Its update of an (n, p) element is one
// sum of 2R products,
//   h' = alpha h + sum_r (beta b_prev_r[n]) (W_x[r][p] x_prev[p])
//                      + (gamma Bbar_r[n]) (W_x[r][p] x[p]),
// the row factors in shared memory ([n][term], read as 16-byte vectors) and
// the column factors in registers; each thread owns VEC columns of every
// ngroups-th row.  At entry the CTA starts 16-byte cp.async copies of the
// lane's whole h (and prev_Bx) into shared memory, so the state is in flight
// while B and C are rotated and the copies hold no registers.  The kernel is
// bound by latency, so occupancy decides its speed: the y partial sums meet
// in warp shuffles and then in the staged state's space once the update has
// read it, and the factored form at rank >= 4 takes two columns per thread
// (the register arrays halve).
// ---------------------------------------------------------------------------
template <int M>
__device__ __forceinline__ void lds_row(const float *p, float (&o)[M]) {
    if constexpr (M % 4 == 0) {
#pragma unroll
        for (int i = 0; i < M / 4; i++) {
            const float4 v = reinterpret_cast<const float4 *>(p)[i];
            o[4 * i] = v.x; o[4 * i + 1] = v.y; o[4 * i + 2] = v.z; o[4 * i + 3] = v.w;
        }
    } else if constexpr (M == 2) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        o[0] = v.x; o[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < M; i++) o[i] = p[i];
    }
}

__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(
                     dst_smem))),
                 "l"(src)
                 : "memory");
}

template <int RT, bool FACT>
struct DecodeGenPlan {
    static constexpr int NV = FACT ? 2 * RT : RT;   // update terms per element
    static constexpr int NS = FACT ? 1 : 2;         // N x P states copied in (h, prev_Bx)
    // columns per thread: 2 for the factored form at rank >= 4, whose column
    // factors (2R x VEC) and y sums (R x VEC) would otherwise hold too many
    // registers for four CTAs per SM
    static constexpr int VEC = (FACT && RT >= 4) ? 2 : 4;
    // y partial sums: one per warp when the lanes of a column share a warp
    static __host__ __device__ int parts(int P, int nt) {
        const int PV = P / VEC;
        return (PV < 32 && (PV & (PV - 1)) == 0) ? nt / 32 : nt / PV;
    }
    // the y partial sums (and the rank sums) reuse the staged state once the
    // update has read it, when they fit there
    static __host__ __device__ bool y_in_state(int N, int P, int nt) {
        return (size_t)(parts(P, nt) + 1) * RT * P <= (size_t)N * P;
    }
    static __host__ __device__ size_t smem_floats(int N, int P, int nt) {
        return (size_t)NS * N * P + (size_t)NV * N + 2 * (size_t)RT * N + N / 2 + 16 * RT +
               (y_in_state(N, P, nt) ? 0 : (size_t)(parts(P, nt) + 1) * RT * P);
    }
};

// NC, PC: dstate and headdim fixed at compile time (0: taken from the
// arguments), so that the row loops unroll fully and the indexing folds.
constexpr int DEC_THREADS = 256;
template <typename T, int RT, bool FACT, int NC, int PC>
__global__ void __launch_bounds__(DEC_THREADS, RT == 1 ? (NC ? 6 : 4) : (RT >= 8 ? 1 : (NC ? (RT >= 4 ? (FACT ? 5 : 2) : 3) : 2)))
    k_decode_gen(DecodeArgs a) {
    using PL = DecodeGenPlan<RT, FACT>;
    constexpr int VEC = PL::VEC, NV = PL::NV, nt = DEC_THREADS;
    using V = typename vecf<VEC>::type;
    const int64_t lane = blockIdx.x, h = lane % a.H;
    const int P = PC ? PC : (int)a.P, N = NC ? NC : (int)a.N, NP2 = N / 2, R = (int)a.R, K = (int)a.K;
    const int tid = threadIdx.x, wid = tid >> 5, ln = tid & 31;
    const int64_t grow = (lane / a.H) * a.G + h / (a.H / a.G);  // the group's B/C rows
    const T *x = static_cast<const T *>(a.x);
    const T *Bg = static_cast<const T *>(a.B) + grow * R * N;
    const T *Cg = static_cast<const T *>(a.C) + grow * R * N;
    T *y = static_cast<T *>(a.y);

    extern __shared__ float4 sm4[];
    float *hs = reinterpret_cast<float *>(sm4);   // N x P   h of this lane (then prev_Bx)
    float *Vs = hs + PL::NS * N * P;              // N x NV  row factors of the update
    float *Cs = Vs + NV * N;                      // N x RT  rotated C, [n][rank]
    float *Bn = Cs + RT * N;                      // RT x N  rotated B (the next b_prev)
    float *phs = Bn + RT * N;                     // N/2     angles of this token
    float *red = phs + N / 2;                     // 16 RT   norm partial sums
    const int npart = PL::parts(P, nt);
    const bool y_in_hs = PL::y_in_state(N, P, nt);
    float *ypart = y_in_hs ? hs : red + 16 * RT;  // npart x RT x P
    float *yr = ypart + npart * RT * P;           // RT x P

    const int PV = P / VEC;              // vectors per state row
    const int ngroups = nt / PV;         // rows streamed concurrently
    const int pv = tid % PV, ng = tid / PV;
    const bool streams = ng < ngroups;
    V *hp = reinterpret_cast<V *>(a.h + lane * (int64_t)N * P) + pv;
    V *up = FACT ? hp : reinterpret_cast<V *>(a.prevBx + lane * (int64_t)N * P) + pv;
    float *us = hs + (FACT ? 0 : N * P);
    {   // the lane's state, 16 bytes per copy, consecutive threads on consecutive bytes
        const float4 *hsrc = reinterpret_cast<const float4 *>(a.h + lane * (int64_t)N * P);
        const float4 *usrc = reinterpret_cast<const float4 *>(a.prevBx + lane * (int64_t)N * P);
        const int nv4 = N * P / 4;
#pragma unroll(NC ? 8 : 4)
        for (int o = tid; o < nv4; o += nt) {
            cp_async16(hs + 4 * o, hsrc + o);
            if (!FACT) cp_async16(us + 4 * o, usrc + o);
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    const float dl = a.dt[lane], lm = a.lam[lane];
    const float al = expf(dl * a.A[h]);
    const float be = (1.f - lm) * dl * al;
    const float ga = lm * dl;

    // column factors: W_x[r][p] x_prev[p] (factored form) and W_x[r][p] x[p]
    float Z[NV][VEC];
    {
        float xv[VEC], xq[VEC];
#pragma unroll
        for (int k = 0; k < VEC; k++) {
            xv[k] = ldf(x, lane * P + pv * VEC + k);
            xq[k] = FACT ? a.xprev[lane * P + pv * VEC + k] : 0.f;
        }
#pragma unroll
        for (int r = 0; r < RT; r++)
#pragma unroll
            for (int k = 0; k < VEC; k++) {
                const int p = pv * VEC + k;
                const float w = r < R ? (a.Wx ? a.Wx[(h * R + r) * P + p] : 1.f) : 0.f;
                if (FACT) {
                    Z[r][k] = w * xq[k];
                    Z[RT + r][k] = w * xv[k];
                } else {
                    Z[r][k] = w * xv[k];
                }
            }
    }

    // QkNorm inverse RMS per rank, every rank in one pass
    float invB[RT], invC[RT];
#pragma unroll
    for (int r = 0; r < RT; r++) { invB[r] = 1.f; invC[r] = 1.f; }
    if (a.nrm.wB || a.nrm.wC) {
        float sb[RT], sc[RT];
#pragma unroll
        for (int r = 0; r < RT; r++) { sb[r] = 0.f; sc[r] = 0.f; }
        for (int it = tid; it < R * N; it += nt) {
            const int r = it / N;
            const float vb = ldf(Bg, it), vc = ldf(Cg, it);
#pragma unroll
            for (int rr = 0; rr < RT; rr++)
                if (rr == r) { sb[rr] += vb * vb; sc[rr] += vc * vc; }
        }
#pragma unroll
        for (int r = 0; r < RT; r++)
            for (int o = 16; o > 0; o >>= 1) {
                sb[r] += __shfl_xor_sync(0xffffffffu, sb[r], o);
                sc[r] += __shfl_xor_sync(0xffffffffu, sc[r], o);
            }
        if (ln == 0)
#pragma unroll
            for (int r = 0; r < RT; r++) { red[(wid * RT + r) * 2] = sb[r]; red[(wid * RT + r) * 2 + 1] = sc[r]; }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < RT; r++) {
            float s = 0.f, c = 0.f;
            for (int w = 0; w < (nt >> 5); w++) { s += red[(w * RT + r) * 2]; c += red[(w * RT + r) * 2 + 1]; }
            invB[r] = rsqrtf(s / N + a.nrm.eps);
            invC[r] = rsqrtf(c / N + a.nrm.eps);
        }
    }

    // one (pair, rank) per thread, rank fastest: every rank's loads in flight
    // at once, and the [n][rank] stores below spread over the banks
    for (int it = tid; it < RT * NP2; it += nt) {
        const int j = it / RT, r = it % RT;
        float b0 = 0.f, b1 = 0.f, c0 = 0.f, c1 = 0.f, q0 = 0.f, q1 = 0.f;
        if (r < R) {
            const int64_t o = r * N + 2 * j;
            b0 = ldf(Bg, o); b1 = ldf(Bg, o + 1); c0 = ldf(Cg, o); c1 = ldf(Cg, o + 1);
            if (FACT) { q0 = a.bprev[lane * R * N + o]; q1 = a.bprev[lane * R * N + o + 1]; }
            float sn = 0.f, cn = 1.f;
            if (j < K) {
                const float phi = a.angle[lane * K + j] + dl * a.theta[lane * K + j];
                if (r == 0) phs[j] = phi;   // written back after every read of the old angle
                sincosf(phi, &sn, &cn);
            }
            float ib = 1.f, ic = 1.f;   // this rank's inverse RMS (selected, not indexed)
#pragma unroll
            for (int rr = 0; rr < RT; rr++)
                if (rr == r) { ib = invB[rr]; ic = invC[rr]; }
            if (a.nrm.wB) { b0 *= ib * a.nrm.wB[2 * j]; b1 *= ib * a.nrm.wB[2 * j + 1]; }
            if (a.nrm.wC) { c0 *= ic * a.nrm.wC[2 * j]; c1 *= ic * a.nrm.wC[2 * j + 1]; }
            const int64_t bo = (h * R + r) * N + 2 * j;
            if (a.nrm.biasB) { b0 += a.nrm.biasB[bo]; b1 += a.nrm.biasB[bo + 1]; }
            if (a.nrm.biasC) { c0 += a.nrm.biasC[bo]; c1 += a.nrm.biasC[bo + 1]; }
            const float rb0 = cn * b0 - sn * b1, rb1 = sn * b0 + cn * b1;
            const float rc0 = cn * c0 - sn * c1, rc1 = sn * c0 + cn * c1;
            b0 = rb0; b1 = rb1; c0 = rc0; c1 = rc1;
        }
        Cs[(2 * j) * RT + r] = c0;
        Cs[(2 * j + 1) * RT + r] = c1;
        if (FACT) {
            Vs[(2 * j) * NV + r] = be * q0;
            Vs[(2 * j + 1) * NV + r] = be * q1;
            Vs[(2 * j) * NV + RT + r] = ga * b0;
            Vs[(2 * j + 1) * NV + RT + r] = ga * b1;
            Bn[r * N + 2 * j] = b0;
            Bn[r * N + 2 * j + 1] = b1;
        } else {
            Vs[(2 * j) * NV + r] = b0;
            Vs[(2 * j + 1) * NV + r] = b1;
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();   // every thread's copies have landed

    float Y[RT][VEC];
#pragma unroll
    for (int r = 0; r < RT; r++)
#pragma unroll
        for (int k = 0; k < VEC; k++) Y[r][k] = 0.f;
    if (streams) {
#pragma unroll(NC ? 8 : 4)
        for (int n = ng; n < N; n += ngroups) {
            float v[NV], c[RT];
            lds_row<NV>(Vs + n * NV, v);
            lds_row<RT>(Cs + n * RT, c);
            float hv[VEC], uv[VEC], ut[VEC];
            vecf<VEC>::unpack(*reinterpret_cast<const V *>(hs + n * P + pv * VEC), hv);
            if (!FACT) vecf<VEC>::unpack(*reinterpret_cast<const V *>(us + n * P + pv * VEC), uv);
#pragma unroll
            for (int k = 0; k < VEC; k++) {
                if (FACT) {
                    float acc = al * hv[k];
#pragma unroll
                    for (int s = 0; s < NV; s++) acc = fmaf(v[s], Z[s][k], acc);
                    hv[k] = acc;
                } else {
                    float u = 0.f;
#pragma unroll
                    for (int r = 0; r < RT; r++) u = fmaf(v[r], Z[r][k], u);
                    ut[k] = u;
                    hv[k] = fmaf(ga, u, fmaf(be, uv[k], al * hv[k]));
                }
            }
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int k = 0; k < VEC; k++) Y[r][k] = fmaf(c[r], hv[k], Y[r][k]);
            hp[n * PV] = vecf<VEC>::pack(hv);
            if (!FACT) up[n * PV] = vecf<VEC>::pack(ut);
        }
    }

    // y: sum the partials over the rows (warp shuffles first where a warp
    // holds whole rows), weight each rank by W_y, add D x
    if (y_in_hs) __syncthreads();   // every thread has read its rows of the staged state
    if (PV < 32 && (PV & (PV - 1)) == 0) {
        for (int o = PV; o < 32; o <<= 1)
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int k = 0; k < VEC; k++) Y[r][k] += __shfl_xor_sync(0xffffffffu, Y[r][k], o);
        if (ln < PV)
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int k = 0; k < VEC; k++) ypart[(wid * RT + r) * P + pv * VEC + k] = Y[r][k];
    } else if (streams) {
#pragma unroll
        for (int r = 0; r < RT; r++)
#pragma unroll
            for (int k = 0; k < VEC; k++) ypart[(ng * RT + r) * P + pv * VEC + k] = Y[r][k];
    }
    __syncthreads();
    const float Dh = a.D[h];
    if (RT == 1 || R == 1) {
        for (int p = tid; p < P; p += nt) {
            float s = 0.f;
            for (int g = 0; g < npart; g++) s += ypart[g * RT * P + p];
            const float xn = ldf(x, lane * P + p);
            stf(y, lane * P + p, (a.Wy ? a.Wy[h * P + p] : 1.f) * s + Dh * xn);
            if (FACT) a.xprev[lane * P + p] = xn;
        }
    } else {
        for (int it = tid; it < R * P; it += nt) {
            const int r = it / P, p = it % P;
            float s = 0.f;
            for (int g = 0; g < npart; g++) s += ypart[(g * RT + r) * P + p];
            yr[it] = (a.Wy ? a.Wy[(h * R + r) * P + p] : 1.f) * s;
        }
        __syncthreads();
        for (int p = tid; p < P; p += nt) {
            float s = 0.f;
            for (int r = 0; r < R; r++) s += yr[r * P + p];
            const float xn = ldf(x, lane * P + p);
            stf(y, lane * P + p, s + Dh * xn);
            if (FACT) a.xprev[lane * P + p] = xn;
        }
    }
    for (int j = tid; j < K; j += nt) a.angle[lane * K + j] = phs[j];
    if (FACT)
        for (int k = tid; k < R * N; k += nt) a.bprev[lane * R * N + k] = Bn[k];
}

template <typename T, int RT, bool FACT, int NC, int PC>
static cudaError_t launch_decode_gen_k(const DecodeArgs &a, cudaStream_t s) {
    // the lane's state is staged in shared memory: up to 64 KB (h) or 128 KB (h and
    // prev_Bx) at dstate x headdim = 16384, past the 48 KB a launch gets by default
    const size_t smem = sizeof(float) * DecodeGenPlan<RT, FACT>::smem_floats((int)a.N, (int)a.P, DEC_THREADS);
    auto kern = k_decode_gen<T, RT, FACT, NC, PC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.Bt * a.H), DEC_THREADS, smem, s>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename T, int RT>
static cudaError_t launch_decode_gen_rt(const DecodeArgs &a, bool factored, cudaStream_t s) {
    // dstate 128 x headdim 64 (the pages' layer shapes) compiled as constants
    if constexpr (RT <= 4)
        if (a.N == 128 && a.P == 64)
            return factored ? launch_decode_gen_k<T, RT, true, 128, 64>(a, s)
                            : launch_decode_gen_k<T, RT, false, 128, 64>(a, s);
    return factored ? launch_decode_gen_k<T, RT, true, 0, 0>(a, s) : launch_decode_gen_k<T, RT, false, 0, 0>(a, s);
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
