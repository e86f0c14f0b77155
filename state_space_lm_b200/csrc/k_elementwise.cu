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
    const int Hi = (int)H;
    // four elements per thread-iteration (16-byte loads and stores); the head
    // of element i is i % H, advanced incrementally instead of divided out
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int hv = (int)((v << 2) % H);
    const int step = (int)((stride << 2) % H);
    for (; v < n4; v += stride) {
        const float4 d = reinterpret_cast<const float4 *>(dt)[v];
        const float4 l = reinterpret_cast<const float4 *>(lam)[v];
        float dd[4] = {d.x, d.y, d.z, d.w}, ll[4] = {l.x, l.y, l.z, l.w};
        float oa[4], ob[4], og[4];
        int hk = hv;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float a = expf(dd[k] * A[hk]);
            oa[k] = a;
            ob[k] = (1.f - ll[k]) * dd[k] * a;
            og[k] = ll[k] * dd[k];
            if (++hk == Hi) hk = 0;
        }
        reinterpret_cast<float4 *>(al)[v] = make_float4(oa[0], oa[1], oa[2], oa[3]);
        reinterpret_cast<float4 *>(be)[v] = make_float4(ob[0], ob[1], ob[2], ob[3]);
        reinterpret_cast<float4 *>(ga)[v] = make_float4(og[0], og[1], og[2], og[3]);
        hv += step;
        if (hv >= Hi) hv -= Hi;
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

// General case (any even N, any K): one CTA per (b, h) lane walks the
// sequence in tiles of ny*SEG tokens.  The
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

// ---- tiled rotation ---------------------------------------------------------
// Eight consecutive elements of a B/C row: one 16-byte vector (bf16) or two
// (fp32).
template <typename T> struct Row8;
template <> struct Row8<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { v = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void get(float *f) const {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; q++) {
            f[2 * q] = __uint_as_float(w[q] << 16);
            f[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void put(__nv_bfloat16 *p, const float *f) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
            w[q] = *reinterpret_cast<uint32_t *>(&h2);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Row8<float> {
    float4 lo, hi;
    __device__ __forceinline__ void load(const float *p) {
        lo = reinterpret_cast<const float4 *>(p)[0];
        hi = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ void zero() { lo = hi = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void get(float *f) const {
        f[0] = lo.x; f[1] = lo.y; f[2] = lo.z; f[3] = lo.w; f[4] = hi.x; f[5] = hi.y; f[6] = hi.z; f[7] = hi.w;
    }
    static __device__ __forceinline__ void put(float *p, const float *f) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
};

// sin/cos of an accumulated angle.  bf16 rows are rounded to 8 bits of
// mantissa on store, so the hardware approximation on the angle reduced mod
// 2 pi (a two-term Cody-Waite split of 2 pi) is ample there; fp32 rows take
// the full-precision sincosf.
__device__ __forceinline__ void sincos_for(const __nv_bfloat16 *, float x, float *s, float *c) {
    const float k = rintf(x * 0.15915494309189535f);
    __sincosf(fmaf(-k, 1.9353071795864769e-3f, fmaf(-k, 6.28125f, x)), s, c);
}
__device__ __forceinline__ void sincos_for(const float *, float x, float *s, float *c) { sincosf(x, s, c); }

// One CTA per (b, h) lane and slice of QS quads (a quad is 4 pairs, 8
// elements of a row).  The lane's tokens go by in tiles of 256 / QS; thread
// (token tr, quad qq) holds one row-quad of the tile.  The angle increments
// dt * theta of a tile are scanned over its tokens -- within a warp by
// shuffles, across the eight warps through shared memory -- on top of the
// angle carried from the previous tile, so every token's angle is the
// sequential sum without a sequential walk.  The next tile's inputs are
// loaded while the current one is rotated (rank 1).  QkNorm needs the whole
// row, so with a norm QS covers all N / 8 quads.  PLAIN (rank 1, no QkNorm,
// no bias) carries none of that code and fits four CTAs per SM, so the
// default workload's 512 CTAs run in one wave.  Needs N % 8 == 0 and K % 4 ==
// 0 (a quad turns wholly or not at all).
template <typename T, int QS, bool PLAIN>
__global__ void __launch_bounds__(256, PLAIN ? 4 : 3) k_rope_tiled(RopeArgs a) {
    constexpr int TT = 256 / QS;
    const int64_t lane = blockIdx.x, b = lane / a.H, h = lane % a.H;
    const int64_t Tn = a.T, H = a.H, G = a.G, hg = h / (H / G);
    const int N = (int)a.N, R = PLAIN ? 1 : (int)a.R, K = (int)a.K;
    const int tid = threadIdx.x, warp = tid >> 5, l32 = tid & 31;
    const int tr = tid / QS, qq = tid % QS;
    const int jq = (int)blockIdx.y * QS + qq;
    const bool turns = 4 * jq < K;
    const T *B = static_cast<const T *>(a.B);
    const T *C = static_cast<const T *>(a.C);
    T *Bo = static_cast<T *>(a.Bo);
    T *Co = static_cast<T *>(a.Co);
    const NormArgs nr = a.nrm;
    const bool has_norm = !PLAIN && (nr.wB || nr.wC), has_bias = !PLAIN && (nr.biasB || nr.biasC);
    __shared__ float4 wt[2][8][QS];      // per-warp angle totals, double-buffered
    __shared__ float4 carry[2][QS];      // angle entering the tile, double-buffered

    if (tr == 0) {
        float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (turns && a.angle0) c0 = *reinterpret_cast<const float4 *>(a.angle0 + lane * K + 4 * jq);
        carry[0][qq] = c0;
        if (Tn == 0 && turns && a.angle_out) *reinterpret_cast<float4 *>(a.angle_out + lane * K + 4 * jq) = c0;
    }
    __syncthreads();

    struct In {
        float dt;
        float4 th;
        Row8<T> rb, rc;                   // rank 1: the B and C row quads, loaded ahead
    };
    auto load_in = [&](int64_t t0, In &in) {
        const int64_t t = t0 + tr;
        in.dt = 0.f;
        in.th = make_float4(0.f, 0.f, 0.f, 0.f);
        in.rb.zero();
        in.rc.zero();
        if (t < Tn) {
            const int64_t bt = (b * Tn + t) * H + h;
            in.dt = a.dt[bt];
            if (turns) in.th = *reinterpret_cast<const float4 *>(a.theta + bt * K + 4 * jq);
            if (R == 1) {
                const int64_t src = ((b * Tn + t) * G + hg) * N + 8 * jq;
                in.rb.load(B + src);
                in.rc.load(C + src);
            }
        }
    };
    In cur, nxt;
    load_in(0, cur);
    int k = 0;
    for (int64_t t0 = 0; t0 < Tn; t0 += TT, k++) {
        load_in(t0 + TT, nxt);
        const int buf = k & 1;
        // inclusive prefix of the increments over the tile's tokens
        float d[4] = {cur.dt * cur.th.x, cur.dt * cur.th.y, cur.dt * cur.th.z, cur.dt * cur.th.w};
#pragma unroll
        for (int off = QS; off < 32; off <<= 1) {
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const float v = __shfl_up_sync(0xffffffffu, d[q], off);
                if (l32 >= off) d[q] += v;
            }
        }
        if (l32 >= 32 - QS) wt[buf][warp][qq] = make_float4(d[0], d[1], d[2], d[3]);
        __syncthreads();
        const float4 cr = carry[buf][qq];
        float phi[4] = {cr.x + d[0], cr.y + d[1], cr.z + d[2], cr.w + d[3]};
#pragma unroll
        for (int w2 = 0; w2 < 7; w2++) {
            if (w2 < warp) {
                const float4 v = wt[buf][w2][qq];
                phi[0] += v.x; phi[1] += v.y; phi[2] += v.z; phi[3] += v.w;
            }
        }
        if (tr == TT - 1) carry[buf ^ 1][qq] = make_float4(phi[0], phi[1], phi[2], phi[3]);
        const int64_t t = t0 + tr;
        float sn[4] = {0.f, 0.f, 0.f, 0.f}, cs[4] = {1.f, 1.f, 1.f, 1.f};
        if (turns) {
#pragma unroll
            for (int q = 0; q < 4; q++) sincos_for(B, phi[q], &sn[q], &cs[q]);
        }
        for (int r = 0; r < R; r++) {
            Row8<T> rb = cur.rb, rc = cur.rc;
            const int64_t src = ((b * Tn + t) * G + hg) * R * N + (int64_t)r * N + 8 * jq;
            if (R > 1) {
                rb.zero();
                rc.zero();
                if (t < Tn) {
                    rb.load(B + src);
                    rc.load(C + src);
                }
            }
            float fb[8], fc[8];
            rb.get(fb);
            rc.get(fc);
            if (has_norm) {
                // inverse RMS of the whole row: the QS lanes of this token hold it
                float sb = 0.f, sc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    sb += fb[e] * fb[e];
                    sc += fc[e] * fc[e];
                }
#pragma unroll
                for (int off = QS / 2; off > 0; off >>= 1) {
                    sb += __shfl_xor_sync(0xffffffffu, sb, off);
                    sc += __shfl_xor_sync(0xffffffffu, sc, off);
                }
                const float ib = nr.wB ? rsqrtf(sb / N + nr.eps) : 1.f, ic = nr.wC ? rsqrtf(sc / N + nr.eps) : 1.f;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    if (nr.wB) fb[e] *= ib * nr.wB[8 * jq + e];
                    if (nr.wC) fc[e] *= ic * nr.wC[8 * jq + e];
                }
            }
            if (has_bias) {
                const int64_t bo = (h * R + r) * N + 8 * jq;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    if (nr.biasB) fb[e] += nr.biasB[bo + e];
                    if (nr.biasC) fc[e] += nr.biasC[bo + e];
                }
            }
            if (turns) {
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const float b0 = fb[2 * q], b1 = fb[2 * q + 1], c0 = fc[2 * q], c1 = fc[2 * q + 1];
                    fb[2 * q] = cs[q] * b0 - sn[q] * b1;
                    fb[2 * q + 1] = sn[q] * b0 + cs[q] * b1;
                    fc[2 * q] = cs[q] * c0 - sn[q] * c1;
                    fc[2 * q + 1] = sn[q] * c0 + cs[q] * c1;
                }
            }
            if (t < Tn) {
                const int64_t dst = (((b * Tn + t) * H + h) * R + r) * N + 8 * jq;
                Row8<T>::put(Bo + dst, fb);
                Row8<T>::put(Co + dst, fc);
            }
        }
        if (t == Tn - 1 && turns && a.angle_out)
            *reinterpret_cast<float4 *>(a.angle_out + lane * K + 4 * jq) = make_float4(phi[0], phi[1], phi[2], phi[3]);
        cur = nxt;
    }
}

template <typename T, bool PLAIN>
static cudaError_t launch_rope_tiled_p(const RopeArgs &a, int qs, cudaStream_t s) {
    const int nq = (int)(a.N / 8);
    const dim3 grid((unsigned)(a.Bt * a.H), (unsigned)(nq / qs));
    switch (qs) {
        case 1: k_rope_tiled<T, 1, PLAIN><<<grid, 256, 0, s>>>(a); break;
        case 2: k_rope_tiled<T, 2, PLAIN><<<grid, 256, 0, s>>>(a); break;
        case 4: k_rope_tiled<T, 4, PLAIN><<<grid, 256, 0, s>>>(a); break;
        case 8: k_rope_tiled<T, 8, PLAIN><<<grid, 256, 0, s>>>(a); break;
        case 16: k_rope_tiled<T, 16, PLAIN><<<grid, 256, 0, s>>>(a); break;
        case 32: k_rope_tiled<T, 32, PLAIN><<<grid, 256, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    count_launch();
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_rope_tiled(const RopeArgs &a, int qs, cudaStream_t s) {
    const bool plain = a.R == 1 && !a.nrm.wB && !a.nrm.wC && !a.nrm.biasB && !a.nrm.biasC;
    return plain ? launch_rope_tiled_p<T, true>(a, qs, s) : launch_rope_tiled_p<T, false>(a, qs, s);
}

// Quads per CTA of the tiled kernel, or 0 when it does not apply: whole quads
// (N % 8 == 0), rotated pairs in whole quads (K % 4 == 0); with QkNorm one
// CTA covers the row, so N / 8 must be a power of two up to 32.
static int rope_tiled_quads(const RopeArgs &a) {
    if (a.N % 8 || a.K % 4) return 0;
    const int nq = (int)(a.N / 8);
    if (a.nrm.wB || a.nrm.wC) return (nq <= 32 && (nq & (nq - 1)) == 0) ? nq : 0;
    return nq % 4 == 0 ? 4 : (nq % 2 == 0 ? 2 : 1);
}

cudaError_t launch_rope(const RopeArgs &a, m3_dtype dt, cudaStream_t s) {
    const int64_t lanes = a.Bt * a.H;
    if (lanes == 0) return cudaSuccess;
    if (const int qs = rope_tiled_quads(a))
        return dt == M3_BF16 ? launch_rope_tiled<__nv_bfloat16>(a, qs, s) : launch_rope_tiled<float>(a, qs, s);
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
