// k_scan_simt.cu -- chunked forward of the Mamba-3 scan on the fp32 FFMA
// pipes (SISO and rank-R MIMO).  This is the path for fp32 inputs, where the
// 1e-5 accuracy bar rules out tensor-core operand rounding, and for shapes
// outside the tensor-core kernel's tile set.
//
// Method (dotLLM pull request, "Stage A: Mamba3SelectiveScan" and the
// streaming-decode comment on shifted_gamma; TorchMamba README, "Math notes":
// chunkwise intra-chunk quadratic part plus an inter-chunk carry):
// with sg_t = (1-lam_{t+1}) dt_{t+1} (0 at the last token) and
// w_t = gamma_t + sg_t, the shifted state g_t = h_t + sg_t U_t obeys the
// two-term recurrence g_t = alpha_t g_{t-1} + w_t U_t, g_{-1} = h0 +
// (1-lam_0) dt_0 prev_Bx0.  Inside a chunk, with cum_t the running sum of
// log alpha from the chunk start,
//   y_t   = e^{cum_t} Cbar_t^T g_in + sum_{s<=t} M[t,s] (Cbar_t . Bbar_s) X_s + D x_t
//   M[t,s] = e^{cum_t - cum_s} w_s for s < t, gamma_t for s = t
//   g_out = e^{cum_end} g_in + sum_s e^{cum_end - cum_s} w_s Bbar_s X_s^T
// For MIMO every token contributes R rows (t, r); the mask depends on the
// tokens only, X_{s,r} = W_x[r] * x_s and y_t = sum_r W_y[r] * Y_{t,r} + D x_t.
//
// Head h reads the B/C rows of group h / (H / G); only the first K pairs
// rotate (partial RoPE), and theta and the angle hold K values per head.
//
// One CTA owns one (b, h) lane and walks its chunks in order; the state g
// (N x P fp32) and the running angle stay in shared memory for the whole
// sequence, so no workspace is used.
#include "m3_internal.cuh"

namespace m3 {

__device__ __forceinline__ float2 ldpair(const float *p, int64_t i) {
    return *reinterpret_cast<const float2 *>(p + i);
}
__device__ __forceinline__ float2 ldpair(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p + i));
}

// Shared-memory footprint in floats (the kernel carves the same regions).
static inline size_t simt_smem_floats(int64_t P, int64_t N, int64_t R, int Q) {
    const size_t QR = (size_t)Q * R, ldn = (size_t)N + 1, NP2 = (size_t)N / 2;
    return (size_t)N * P + 2 * QR * ldn + QR * P + QR * QR + (size_t)Q * NP2 + 6 * (size_t)Q +
           2 * QR + NP2 + 32;
}

size_t scan_simt_smem_bytes(int64_t P, int64_t N, int64_t R, int Q) {
    return sizeof(float) * simt_smem_floats(P, N, R, Q);
}

// Largest chunk <= the requested one whose working set fits shared memory.
int scan_simt_chunk(int64_t P, int64_t N, int64_t R, int64_t chunk) {
    const size_t limit = 200 * 1024;
    int q = (int)(chunk < 256 ? chunk : 256);
    while (q > 1 && scan_simt_smem_bytes(P, N, R, q) > limit) q = (q + 1) / 2;
    if (scan_simt_smem_bytes(P, N, R, q) > limit) return 0;
    return q;
}

template <typename T>
__global__ void __launch_bounds__(256) k_scan_simt(ScanArgs a) {
    const int64_t lane = blockIdx.x, b = lane / a.H, h = lane % a.H;
    const int64_t Tn = a.T, H = a.H, G = a.G, hg = h / (H / G);
    const int P = (int)a.P, N = (int)a.N, R = (int)a.R, Q = a.Q, K = (int)a.K;
    const int NP2 = N / 2, ldn = N + 1, QR = Q * R;
    const int64_t NPs = (int64_t)N * P;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int warp = tid >> 5, l32 = tid & 31, nw = nt >> 5;
    const T *x = static_cast<const T *>(a.x);
    const T *Bg = static_cast<const T *>(a.B);
    const T *Cg = static_cast<const T *>(a.C);
    T *y = static_cast<T *>(a.y);
    const float Ah = a.A[h], Dh = a.D[h];

    extern __shared__ float sm[];
    float *g = sm;                       // N*P      shifted state
    float *Bb = g + NPs;                 // QR*ldn   rotated B rows
    float *Cb = Bb + (size_t)QR * ldn;   // QR*ldn   rotated C rows
    float *X = Cb + (size_t)QR * ldn;    // QR*P     W_x * x rows
    float *S = X + (size_t)QR * P;       // QR*QR    masked scores
    float *Ph = S + (size_t)QR * QR;     // Q*K      angles (Q*NP2 reserved)
    float *cum = Ph + (size_t)Q * NP2;   // Q
    float *w = cum + Q;                  // Q
    float *gam = w + Q;                  // Q
    float *cs = gam + Q;                 // Q        e^{cum_end - cum_s} w_s
    float *ec = cs + Q;                  // Q        e^{cum_t}
    float *dts = ec + Q;                 // Q
    float *invB = dts + Q;               // QR
    float *invC = invB + QR;             // QR
    float *phi = invC + QR;              // K        running angle

    for (int j = tid; j < K; j += nt) phi[j] = a.angle0 ? a.angle0[lane * K + j] : 0.f;
    float f0 = 0.f;
    if (Tn > 0) {
        const int64_t i0 = (b * Tn) * H + h;
        f0 = (1.f - a.lam[i0]) * a.dt[i0];
    }
    for (int64_t k = tid; k < NPs; k += nt)
        g[k] = (a.h0 ? a.h0[lane * NPs + k] : 0.f) +
               f0 * (a.prevBx0 ? a.prevBx0[lane * NPs + k] : 0.f);
    __syncthreads();

    for (int64_t t0 = 0; t0 < Tn; t0 += Q) {
        const int L = (int)((Tn - t0) < Q ? (Tn - t0) : Q);
        const int LR = L * R;
        // (a) per-token coefficients
        for (int i = tid; i < L; i += nt) {
            const int64_t bt = (b * Tn + t0 + i) * H + h;
            const float dl = a.dt[bt], lm = a.lam[bt];
            float sg = 0.f;
            if (t0 + i + 1 < Tn) {
                const int64_t nx = bt + H;
                sg = (1.f - a.lam[nx]) * a.dt[nx];
            }
            dts[i] = dl;
            cum[i] = dl * Ah;
            gam[i] = lm * dl;
            w[i] = lm * dl + sg;
        }
        // QkNorm: inverse RMS of every B and C row of the chunk
        if (a.nrm.wB || a.nrm.wC) {
            for (int row = warp; row < LR; row += nw) {
                const int64_t base = (((b * Tn + t0 + row / R) * G + hg) * R + row % R) * N;
                float sb = 0.f, sc = 0.f;
                for (int n = l32; n < N; n += 32) {
                    const float vb = ldf(Bg, base + n), vc = ldf(Cg, base + n);
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
        if (tid == 0) {
            float run = 0.f;
            for (int i = 0; i < L; i++) {
                run += cum[i];
                cum[i] = run;
            }
        }
        __syncthreads();
        for (int i = tid; i < L; i += nt) {
            cs[i] = expf(cum[L - 1] - cum[i]) * w[i];
            ec[i] = expf(cum[i]);
        }
        // (b) running angle per pair over the chunk's tokens
        for (int j = tid; j < K; j += nt) {
            float c = phi[j];
            for (int i = 0; i < L; i++) {
                c += dts[i] * a.theta[((b * Tn + t0 + i) * H + h) * K + j];
                Ph[i * K + j] = c;
            }
            phi[j] = c;
        }
        __syncthreads();
        // (c) QkNorm gain, bias and rotation of every B and C row
        for (int it = tid; it < LR * NP2; it += nt) {
            const int j = it % NP2, row = it / NP2, i = row / R, r = row % R;
            const int64_t base = (((b * Tn + t0 + i) * G + hg) * R + r) * N + 2 * j;
            float2 bv = ldpair(Bg, base), cv = ldpair(Cg, base);
            if (a.nrm.wB) {
                bv.x *= invB[row] * a.nrm.wB[2 * j];
                bv.y *= invB[row] * a.nrm.wB[2 * j + 1];
            }
            if (a.nrm.wC) {
                cv.x *= invC[row] * a.nrm.wC[2 * j];
                cv.y *= invC[row] * a.nrm.wC[2 * j + 1];
            }
            if (a.nrm.biasB) {
                bv.x += a.nrm.biasB[(h * R + r) * N + 2 * j];
                bv.y += a.nrm.biasB[(h * R + r) * N + 2 * j + 1];
            }
            if (a.nrm.biasC) {
                cv.x += a.nrm.biasC[(h * R + r) * N + 2 * j];
                cv.y += a.nrm.biasC[(h * R + r) * N + 2 * j + 1];
            }
            float sn = 0.f, cn = 1.f;
            if (j < K) sincosf(Ph[i * K + j], &sn, &cn);
            Bb[row * ldn + 2 * j] = cn * bv.x - sn * bv.y;
            Bb[row * ldn + 2 * j + 1] = sn * bv.x + cn * bv.y;
            Cb[row * ldn + 2 * j] = cn * cv.x - sn * cv.y;
            Cb[row * ldn + 2 * j + 1] = sn * cv.x + cn * cv.y;
        }
        for (int it = tid; it < LR * P; it += nt) {
            const int p = it % P, row = it / P, i = row / R, r = row % R;
            const float xv = ldf(x, ((b * Tn + t0 + i) * H + h) * P + p);
            X[row * P + p] = (a.Wx ? a.Wx[(h * R + r) * P + p] : 1.f) * xv;
        }
        __syncthreads();
        // (d) masked scores S[(t,r'), (s,r)] for s <= t
        for (int it = tid; it < LR * LR; it += nt) {
            const int cr = it % LR, rr = it / LR, tt = rr / R, ss = cr / R;
            float v = 0.f;
            if (ss <= tt) {
                float dot = 0.f;
                const float *cp = Cb + rr * ldn, *bp = Bb + cr * ldn;
                for (int n = 0; n < N; n++) dot += cp[n] * bp[n];
                const float coef = (ss == tt) ? gam[tt] : expf(cum[tt] - cum[ss]) * w[ss];
                v = dot * coef;
            }
            S[rr * LR + cr] = v;
        }
        __syncthreads();
        // (e) outputs of the chunk
        for (int it = tid; it < L * P; it += nt) {
            const int p = it % P, i = it / P;
            float acc = 0.f;
            for (int r2 = 0; r2 < R; r2++) {
                const int row = i * R + r2;
                float yi = 0.f;
                const float *sp = S + row * LR;
                for (int cr = 0; cr < (i + 1) * R; cr++) yi += sp[cr] * X[cr * P + p];
                float yg = 0.f;
                const float *cp = Cb + row * ldn;
                for (int n = 0; n < N; n++) yg += cp[n] * g[n * P + p];
                acc += (a.Wy ? a.Wy[(h * R + r2) * P + p] : 1.f) * (yi + ec[i] * yg);
            }
            const int64_t xi = ((b * Tn + t0 + i) * H + h) * P + p;
            stf(y, xi, acc + Dh * ldf(x, xi));
        }
        __syncthreads();
        // (f) carry the shifted state to the end of the chunk
        for (int64_t it = tid; it < NPs; it += nt) {
            const int p = (int)(it % P), n = (int)(it / P);
            float acc = ec[L - 1] * g[it];
            for (int cr = 0; cr < LR; cr++) acc += cs[cr / R] * Bb[cr * ldn + n] * X[cr * P + p];
            g[it] = acc;
        }
        if (t0 + L == Tn && a.prevBx_out) {
            for (int64_t it = tid; it < NPs; it += nt) {
                const int p = (int)(it % P), n = (int)(it / P);
                float u = 0.f;
                for (int r = 0; r < R; r++)
                    u += Bb[((L - 1) * R + r) * ldn + n] * X[((L - 1) * R + r) * P + p];
                a.prevBx_out[lane * NPs + it] = u;
            }
        }
        __syncthreads();
    }
    // the shifted state after the last token equals h_{T-1} (no lookahead)
    if (a.h_out)
        for (int64_t k = tid; k < NPs; k += nt) a.h_out[lane * NPs + k] = g[k];
    if (Tn == 0 && a.prevBx_out)
        for (int64_t k = tid; k < NPs; k += nt)
            a.prevBx_out[lane * NPs + k] = a.prevBx0 ? a.prevBx0[lane * NPs + k] : 0.f;
    if (a.angle_out)
        for (int j = tid; j < K; j += nt) a.angle_out[lane * K + j] = phi[j];
}

cudaError_t launch_scan_simt(const ScanArgs &a, m3_dtype dt, cudaStream_t s) {
    const int64_t lanes = a.Bt * a.H;
    if (lanes == 0) return cudaSuccess;
    const size_t smem = scan_simt_smem_bytes(a.P, a.N, a.R, a.Q);
    if (dt == M3_BF16) {
        cudaFuncSetAttribute(k_scan_simt<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        k_scan_simt<__nv_bfloat16><<<(unsigned)lanes, 256, smem, s>>>(a);
    } else {
        cudaFuncSetAttribute(k_scan_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_scan_simt<float><<<(unsigned)lanes, 256, smem, s>>>(a);
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace m3
