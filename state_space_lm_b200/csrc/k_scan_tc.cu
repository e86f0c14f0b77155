// k_scan_tc.cu -- SISO chunked forward of the Mamba-3 scan on the sm_100a
// tensor cores (bf16 inputs, headdim 64, dState 128, chunk 64).
//
// The method is the chunked form of the trapezoidal recurrence (dotLLM pull
// request, "Stage A: Mamba3SelectiveScan" and the streaming-decode comment:
// shifted_gamma[t] = DT[t+1](1-trap[t+1]), scale = gamma + shifted_gamma,
// boundary fold DT[0](1-trap[0]); TorchMamba README, "Math notes": Mamba-2
// chunkwise intra-chunk quadratic part plus inter-chunk carry, and Props. 2-4
// for the data-dependent rotation).  With sg_t = (1-lam_{t+1}) dt_{t+1},
// w_t = gamma_t + sg_t and the shifted state g_t = h_t + sg_t U_t:
//   g_t = alpha_t g_{t-1} + w_t U_t,    g_{-1} = h0 + (1-lam_0) dt_0 prev_Bx0
// and inside a chunk (cum_t = sum of log alpha from the chunk start):
//   y_t   = e^{cum_t} Cbar_t^T g_in + sum_{s<=t} M[t,s] (Cbar_t . Bbar_s) x_s + D x_t
//   g_out = e^{cum_end} g_in + sum_s e^{cum_end - cum_s} w_s Bbar_s x_s^T
// with M[t,s] = e^{cum_t - cum_s} w_s (s < t), gamma_t (s = t).
//
// One CTA owns one (b, h) lane and walks its chunks in order.  Per chunk four
// UMMAs (tcgen05.mma kind::f16, bf16 operands in shared memory, fp32
// accumulators in tensor memory):
//   D1 = Cbar . Bsc^T             scores            M=64  N=64  K=128
//   D3 = Cbar . g_in              inter-chunk term  M=64  N=64  K=128
//   D2 = S' . X                   intra-chunk term  M=64  N=64  K=64
//   D4 = Bsc^T . Xw               chunk state       M=128 N=64  K=64
// The decay mask is split into a row factor and a column factor: Bsc holds
// e_s Bbar_s with e_s = e^{cum_end - cum_s}, the masking multiplies row t by
// r_t = e^{cum_t - cum_end} and column s by w_s (gamma_t on the diagonal), and
// Xw holds w_s x_s, so D4 is the chunk's state contribution directly.  When a
// chunk's log-decay range exceeds 60 the factors could leave the fp32 range;
// such a chunk uses Bsc = Bbar, an exact per-element mask
// e^{cum_t - cum_s} w_s and Xw = e^{cum_end - cum_s} w_s x_s instead.
//
// Warp roles (12 warps): 0 TMA producer, 1 MMA issuer (and TMEM owner),
// 2 per-token coefficients, 3 Xw scaling, 4-7 rotation (QkNorm, bias, RoPE),
// 8-11 epilogue (TMEM -> masked scores, outputs, fp32 state in registers).
// Every wait is bounded: past ~1 s the kernel records an error, stops issuing
// work, drains what it has in flight and returns.
#include <cuda.h>

#include "m3_internal.cuh"

namespace m3 {
namespace tc {

constexpr int Q = 64, P = 64, N = 128, NP2 = 64;
constexpr int THREADS = 384;
constexpr int W_TMA = 0, W_MMA = 1, W_COEF = 2, W_XW = 3, W_PREP0 = 4, W_EPI0 = 8;

// ---- shared-memory map (bytes from a 1024-aligned base) ------------------
constexpr int SZ_X = Q * P * 2;          // 8 KB, bf16, 128B-swizzled (TMA)
constexpr int SZ_BC = Q * N * 2;         // 16 KB, bf16, row-major (TMA)
constexpr int SZ_TH = Q * NP2 * 4;       // 16 KB, fp32, row-major (TMA)
constexpr int STAGE = SZ_X + 2 * SZ_BC + SZ_TH;
constexpr int OFF_STAGE0 = 0;
constexpr int OFF_BSC = 2 * STAGE;               // [2 atoms][Q][64] bf16, SW128
constexpr int OFF_CB = OFF_BSC + Q * N * 2;      // [2 atoms][Q][64] bf16, SW128
constexpr int OFF_SP = OFF_CB + Q * N * 2;       // [Q][Q] bf16, SW128
constexpr int OFF_XW = OFF_SP + Q * Q * 2;       // [Q][P] bf16, SW128
constexpr int OFF_GB = OFF_XW + Q * P * 2;       // [N][P] bf16, SW128
constexpr int OFF_YT = OFF_GB + N * P * 2;       // [Q][P] bf16, SW128
constexpr int OFF_COEF = OFF_YT + Q * P * 2;
// per-chunk coefficient buffer (double-buffered), floats
constexpr int CF_W = 0, CF_GAM = Q, CF_E = 2 * Q, CF_R = 3 * Q, CF_EC = 4 * Q, CF_XS = 5 * Q,
              CF_C2 = 6 * Q, CF_DT = 7 * Q, CF_SCAL = 8 * Q, CF_FLOATS = 8 * Q + 8;
constexpr int OFF_BLAST = OFF_COEF + 2 * CF_FLOATS * 4;  // fp32 [N]
constexpr int OFF_PHIC = OFF_BLAST + N * 4;              // fp32 [NP2] running angle
constexpr int OFF_PART = OFF_PHIC + NP2 * 4;             // fp32 [NP2] half-chunk angle sums
constexpr int OFF_INV = OFF_PART + NP2 * 4;              // fp32 [2][Q] QkNorm inverse RMS
constexpr int OFF_BAR = OFF_INV + 2 * Q * 4;             // mbarriers
constexpr int NBAR = 18;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;             // tmem slot, abort flag
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;         // + alignment slack

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_CFULL0, B_CFULL1, B_CEMPTY0, B_CEMPTY1,
    B_OPSREADY, B_OPSFREE, B_SFULL, B_STAKEN, B_SPFULL, B_YFULL, B_YTAKEN, B_STFULL, B_STTAKEN,
    B_DRAIN
};

constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_D1 = 0, COL_D2 = 64, COL_D3 = 128, COL_D4 = 192;

struct TcArgs {
    const float *dt, *A, *lam, *D;
    const float *h0, *prevBx0, *angle0;
    NormArgs nrm;
    float *h_out, *prevBx_out, *angle_out;
    int64_t Bt, T, H;
    int *err;
};

// ---- PTX wrappers ---------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

constexpr long long WAIT_LIMIT_CYCLES = 2000000000LL;  // ~1 s at 1.9 GHz

// Bounded wait on an mbarrier phase.  Returns false when the kernel is
// aborting (this wait timed out, or another thread's did).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                         int site) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
            *abort_flag = 1;
            atomicCAS(err, 0, site);
            return false;
        }
    }
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// Named barrier that also ORs a predicate over the participating threads, so
// that every thread of a group takes the same decision.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void tma_load4(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(dst),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_store4(const CUtensorMap *map, int c0, int c1, int c2, int c3, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(map),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// UMMA shared-memory descriptor, 128B swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// Instruction descriptor: kind::f16, bf16 x bf16 -> fp32, dense.
__host__ __device__ constexpr uint32_t idesc(int M, int Nn, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(Nn >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t dtmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
            dtmem),
        "l"(a), "l"(b), "r"(id), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    __syncwarp();   // .sync.aligned: the whole warp issues it together
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() {
    __syncwarp();
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return __bfloat1622float2(v);
}
// byte offset of element col (0..63) in row `row` of a 128B-swizzled tile
// whose rows are 128 bytes (64 bf16) -- 16-byte chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sw128(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7)) << 4) | ((col & 7) << 1)));
}

// sin/cos with Cody-Waite reduction to [-pi, pi] (2 pi split into an exactly
// representable head and a tail), then the hardware approximation there.
__device__ __forceinline__ void sincos_rr(float x, float *s, float *c) {
    const float k = rintf(x * 0.15915494309189535f);
    float r = fmaf(-k, 6.28125f, x);
    r = fmaf(-k, 1.9353071795864769e-3f, r);
    __sincosf(r, s, c);
}

__global__ void __launch_bounds__(THREADS, 1)
    k_scan_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
              const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_th,
              const __grid_constant__ CUtensorMap map_y, TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, l32 = tid & 31;
    const int64_t lane_id = blockIdx.x, b = lane_id / a.H, h = lane_id % a.H;
    const int64_t Tn = a.T, H = a.H;
    const int nchunks = (int)((Tn + Q - 1) / Q);
    auto bar = [&](int i) { return sbase + OFF_BAR + 8 * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    float *coef0 = reinterpret_cast<float *>(sm + OFF_COEF);
    float *blast = reinterpret_cast<float *>(sm + OFF_BLAST);
    float *phic = reinterpret_cast<float *>(sm + OFF_PHIC);
    float *part = reinterpret_cast<float *>(sm + OFF_PART);
    float *inv = reinterpret_cast<float *>(sm + OFF_INV);

    if (tid == 0) {
        const uint32_t counts[NBAR] = {1, 1, 4, 4, 1, 1, 3, 3, 2, 1, 1, 4, 4, 1, 4, 1, 4, 1};
        for (int i = 0; i < NBAR; i++) mbar_init(bar(i), counts[i]);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_x) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_b) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_c) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_th) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_y) : "memory");
    }
    if (warp == W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid < NP2) phic[tid] = a.angle0 ? a.angle0[lane_id * NP2 + tid] : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // ------------------------------------------------------------ producer
        if (l32 == 0) {
            int issued = 0;
            for (int c = 0; c < nchunks; c++) {
                const int s = c & 1, k = c >> 1;
                if (k > 0 && !wait_bar(bar(B_EMPTY0 + s), (k - 1) & 1, abort_flag, a.err, 1)) break;
                const uint32_t st = sbase + OFF_STAGE0 + s * STAGE;
                const uint32_t fb = bar(B_FULL0 + s);
                mbar_expect_tx(fb, STAGE);
                const int t0 = c * Q;
                tma_load4(st, &map_x, 0, (int)h, t0, (int)b, fb);
                tma_load4(st + SZ_X, &map_b, 0, (int)h, t0, (int)b, fb);
                tma_load4(st + SZ_X + SZ_BC, &map_c, 0, (int)h, t0, (int)b, fb);
                tma_load4(st + SZ_X + 2 * SZ_BC, &map_th, 0, (int)h, t0, (int)b, fb);
                issued = c + 1;
            }
            // never leave loads in flight into shared memory at exit
            for (int c = (issued > 2 ? issued - 2 : 0); c < issued; c++) {
                const long long t0 = clock64();
                while (!mbar_try(bar(B_FULL0 + (c & 1)), (c >> 1) & 1) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
                }
            }
        }
    } else if (warp == W_COEF) {
        // --------------------------------------------------------- coefficients
        const float L2E = 1.4426950408889634f;
        const float A2 = a.A[h] * L2E;
        const float UNSAFE2 = 60.f * L2E;
        for (int c = 0; c < nchunks; c++) {
            const int s = c & 1, k = c >> 1;
            int ok = 1;
            if (l32 == 0 && k > 0) ok = wait_bar(bar(B_CEMPTY0 + s), (k - 1) & 1, abort_flag, a.err, 2);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            float *cf = coef0 + s * CF_FLOATS;
            const int64_t t0 = (int64_t)c * Q;
            const int L = (int)((Tn - t0) < Q ? (Tn - t0) : Q);
            float la[2], wv[2], gv[2], dv[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i = l32 + 32 * u;
                la[u] = wv[u] = gv[u] = dv[u] = 0.f;
                if (i < L) {
                    const int64_t bt = (b * Tn + t0 + i) * H + h;
                    const float dl = a.dt[bt], lm = a.lam[bt];
                    float sg = 0.f;
                    if (t0 + i + 1 < Tn) sg = (1.f - a.lam[bt + H]) * a.dt[bt + H];
                    gv[u] = lm * dl;
                    wv[u] = gv[u] + sg;
                    la[u] = dl * A2;
                    dv[u] = dl;
                }
            }
            // inclusive scan of log2(alpha) over the 64 tokens
#pragma unroll
            for (int u = 0; u < 2; u++)
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, la[u], o);
                    if (l32 >= o) la[u] += v;
                }
            la[1] += __shfl_sync(0xffffffffu, la[0], 31);
            const float cend = __shfl_sync(0xffffffffu, (L - 1) < 32 ? la[0] : la[1], (L - 1) & 31);
            float dev = 0.f;
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i = l32 + 32 * u;
                if (i >= L) la[u] = cend;
                dev = fmaxf(dev, fabsf(la[u] - cend));
            }
            const bool unsafe = __any_sync(0xffffffffu, dev > UNSAFE2);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i = l32 + 32 * u;
                const float e = exp2f(cend - la[u]);
                cf[CF_W + i] = wv[u];
                cf[CF_GAM + i] = gv[u];
                cf[CF_E + i] = unsafe ? 1.f : e;
                cf[CF_R + i] = exp2f(la[u] - cend);
                cf[CF_EC + i] = exp2f(la[u]);
                cf[CF_XS + i] = unsafe ? e * wv[u] : wv[u];
                cf[CF_C2 + i] = la[u];
                cf[CF_DT + i] = dv[u];
            }
            if (l32 == 0) {
                cf[CF_SCAL + 0] = exp2f(cend);
                cf[CF_SCAL + 1] = unsafe ? 1.f : 0.f;
                cf[CF_SCAL + 2] = (float)L;
            }
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_CFULL0 + s));
        }
    } else if (warp == W_XW) {
        // ------------------------------------------------- Xw = diag(xs) . X
        for (int c = 0; c < nchunks; c++) {
            const int s = c & 1, k = c >> 1;
            int ok = 1;
            if (l32 == 0) {
                ok = wait_bar(bar(B_FULL0 + s), k & 1, abort_flag, a.err, 3) &&
                     wait_bar(bar(B_CFULL0 + s), k & 1, abort_flag, a.err, 4) &&
                     (c == 0 || wait_bar(bar(B_OPSFREE), (c - 1) & 1, abort_flag, a.err, 5));
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const float *cf = coef0 + s * CF_FLOATS;
            const uint4 *src = reinterpret_cast<const uint4 *>(sm + OFF_STAGE0 + s * STAGE);
            uint4 *dst = reinterpret_cast<uint4 *>(sm + OFF_XW);
#pragma unroll 4
            for (int v = l32; v < Q * P / 8; v += 32) {
                const float sc = cf[CF_XS + (v >> 3)];   // 8 vectors per 128-byte row
                uint4 d = src[v];
                uint32_t *w = reinterpret_cast<uint32_t *>(&d);
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const float2 f = unpack_bf16(w[q]);
                    w[q] = pack_bf16(f.x * sc, f.y * sc);
                }
                dst[v] = d;
            }
            fence_async_smem();
            __syncwarp();
            if (l32 == 0) {
                mbar_arrive(bar(B_OPSREADY));
                mbar_arrive(bar(B_EMPTY0 + s));
                mbar_arrive(bar(B_CEMPTY0 + s));
            }
        }
    } else if (warp >= W_PREP0 && warp < W_PREP0 + 4) {
        // ----------------------------------- QkNorm + bias + RoPE rotation
        const int pt = tid - W_PREP0 * 32;         // 0..127
        const int j = pt & 63, half = pt >> 6;     // pair, token half
        const NormArgs nr = a.nrm;
        const bool has_norm = nr.wB || nr.wC;
        const float wb0 = nr.wB ? nr.wB[2 * j] : 1.f, wb1 = nr.wB ? nr.wB[2 * j + 1] : 1.f;
        const float wc0 = nr.wC ? nr.wC[2 * j] : 1.f, wc1 = nr.wC ? nr.wC[2 * j + 1] : 1.f;
        const float bb0 = nr.biasB ? nr.biasB[h * N + 2 * j] : 0.f, bb1 = nr.biasB ? nr.biasB[h * N + 2 * j + 1] : 0.f;
        const float bc0 = nr.biasC ? nr.biasC[h * N + 2 * j] : 0.f, bc1 = nr.biasC ? nr.biasC[h * N + 2 * j + 1] : 0.f;
        uint8_t *bsc = sm + OFF_BSC;
        uint8_t *cb = sm + OFF_CB;
        // element (row i, n) of the two-atom [n/64][row][64] 128B-swizzled tiles
        const uint32_t atom = (uint32_t)(j >> 5) * (Q * 128);
        const int col = (2 * j) & 63;
        for (int c = 0; c < nchunks; c++) {
            const int s = c & 1, k = c >> 1;
            bool fail = false;
            if (pt == 0) {
                fail = !(wait_bar(bar(B_FULL0 + s), k & 1, abort_flag, a.err, 6) &&
                         wait_bar(bar(B_CFULL0 + s), k & 1, abort_flag, a.err, 7) &&
                         (c == 0 || wait_bar(bar(B_OPSFREE), (c - 1) & 1, abort_flag, a.err, 8)));
            }
            if (named_bar_or(1, 128, fail)) break;
            const float *cf = coef0 + s * CF_FLOATS;
            const uint8_t *stg = sm + OFF_STAGE0 + s * STAGE;
            const uint32_t *braw = reinterpret_cast<const uint32_t *>(stg + SZ_X);
            const uint32_t *craw = reinterpret_cast<const uint32_t *>(stg + SZ_X + SZ_BC);
            const float *th = reinterpret_cast<const float *>(stg + SZ_X + 2 * SZ_BC);
            const int L = (int)cf[CF_SCAL + 2];
            if (has_norm) {
                // inverse RMS of each B and C row of the chunk: one warp per row
                const int wp = pt >> 5;
                for (int r = wp; r < 2 * Q; r += 4) {
                    const int i = r & (Q - 1);
                    const uint32_t *raw = (r < Q) ? braw : craw;
                    float ss = 0.f;
                    for (int q = l32; q < NP2; q += 32) {
                        const float2 f = unpack_bf16(raw[i * NP2 + q]);
                        ss += f.x * f.x + f.y * f.y;
                    }
                    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    if (l32 == 0) inv[r] = rsqrtf(ss / N + nr.eps);
                }
            }
            // pass 1: angle increments of my half of the chunk
            float acc = 0.f;
            const int i0 = half * 32;
            for (int i = i0; i < i0 + 32; i++) acc += cf[CF_DT + i] * th[i * NP2 + j];
            if (half == 0) part[j] = acc;
            named_bar(1, 128);
            float phi = phic[j] + (half ? part[j] : 0.f);
            // pass 2: rotate
            const bool last_chunk = (c == nchunks - 1);
            for (int i = i0; i < i0 + 32; i++) {
                uint32_t pb = 0u, pc = 0u;
                if (i < L) {
                    phi = fmaf(cf[CF_DT + i], th[i * NP2 + j], phi);
                    float sn, cs;
                    sincos_rr(phi, &sn, &cs);
                    float2 bv = unpack_bf16(braw[i * NP2 + j]);
                    float2 cv = unpack_bf16(craw[i * NP2 + j]);
                    if (has_norm) {
                        if (nr.wB) { bv.x *= inv[i] * wb0; bv.y *= inv[i] * wb1; }
                        if (nr.wC) { cv.x *= inv[Q + i] * wc0; cv.y *= inv[Q + i] * wc1; }
                    }
                    bv.x += bb0; bv.y += bb1;
                    cv.x += bc0; cv.y += bc1;
                    const float rb0 = cs * bv.x - sn * bv.y, rb1 = sn * bv.x + cs * bv.y;
                    const float rc0 = cs * cv.x - sn * cv.y, rc1 = sn * cv.x + cs * cv.y;
                    const float e = cf[CF_E + i];
                    pb = pack_bf16(rb0 * e, rb1 * e);
                    pc = pack_bf16(rc0, rc1);
                    if (last_chunk && i == L - 1) {
                        blast[2 * j] = rb0;
                        blast[2 * j + 1] = rb1;
                    }
                }
                *reinterpret_cast<uint32_t *>(bsc + atom + sw128(i, col)) = pb;
                *reinterpret_cast<uint32_t *>(cb + atom + sw128(i, col)) = pc;
            }
            fence_async_smem();
            named_bar(1, 128);
            if (half == 1) {
                phic[j] = phi;      // the angle after the chunk's last token
                if (last_chunk && a.angle_out) a.angle_out[lane_id * NP2 + j] = phi;
            }
            if (pt == 0) {
                mbar_arrive(bar(B_OPSREADY));
                mbar_arrive(bar(B_EMPTY0 + s));
                mbar_arrive(bar(B_CEMPTY0 + s));
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issue
        if (l32 == 0) {
            const uint32_t id_kk = idesc(64, 64, 0, 0);    // D1 = Cbar . Bsc^T
            const uint32_t id_kmn = idesc(64, 64, 0, 1);   // D2, D3: B operand MN-major
            const uint32_t id_st = idesc(128, 64, 1, 1);   // D4: A and B MN-major
            const uint32_t a_bsc = sbase + OFF_BSC, a_cb = sbase + OFF_CB, a_sp = sbase + OFF_SP;
            const uint32_t a_xw = sbase + OFF_XW, a_gb = sbase + OFF_GB;
            for (int c = 0; c < nchunks; c++) {
                const int s = c & 1;
                const uint32_t a_x = sbase + OFF_STAGE0 + s * STAGE;
                if (!wait_bar(bar(B_OPSREADY), c & 1, abort_flag, a.err, 10)) break;
                if (c > 0 && !wait_bar(bar(B_STAKEN), (c - 1) & 1, abort_flag, a.err, 11)) break;
                tc_fence_after();
                for (int kk = 0; kk < N / 16; kk++) {
                    const uint32_t off = (kk >> 2) * (Q * 128) + (kk & 3) * 32;
                    umma(tmem + COL_D1, sdesc(a_cb + off, 16, 1024), sdesc(a_bsc + off, 16, 1024), id_kk, kk > 0);
                }
                umma_commit(bar(B_SFULL));
                if (!wait_bar(bar(B_STTAKEN), c & 1, abort_flag, a.err, 12)) break;
                tc_fence_after();
                for (int kk = 0; kk < Q / 16; kk++)
                    umma(tmem + COL_D4, sdesc(a_bsc + kk * 2048, Q * 128, 1024), sdesc(a_xw + kk * 2048, Q * 128, 1024),
                         id_st, kk > 0);
                umma_commit(bar(B_STFULL));
                if (c > 0 && !wait_bar(bar(B_YTAKEN), (c - 1) & 1, abort_flag, a.err, 13)) break;
                tc_fence_after();
                for (int kk = 0; kk < N / 16; kk++) {
                    const uint32_t off = (kk >> 2) * (Q * 128) + (kk & 3) * 32;
                    umma(tmem + COL_D3, sdesc(a_cb + off, 16, 1024), sdesc(a_gb + kk * 2048, N * 128, 1024), id_kmn,
                         kk > 0);
                }
                umma_commit(bar(B_OPSFREE));
                if (!wait_bar(bar(B_SPFULL), c & 1, abort_flag, a.err, 14)) break;
                tc_fence_after();
                for (int kk = 0; kk < Q / 16; kk++)
                    umma(tmem + COL_D2, sdesc(a_sp + kk * 32, 16, 1024), sdesc(a_x + kk * 2048, Q * 128, 1024), id_kmn,
                         kk > 0);
                umma_commit(bar(B_YFULL));
                umma_commit(bar(B_EMPTY0 + s));
            }
            // drain: every MMA issued so far has completed before TMEM is freed
            umma_commit(bar(B_DRAIN));
            const long long t0 = clock64();
            while (!mbar_try(bar(B_DRAIN), 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const int q = warp & 3;                      // TMEM lane quarter
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const int n = 32 * q + l32;                  // state row owned by this thread
        const int trow = 16 * q + l32;               // score/output row (valid for l32 < 16)
        const bool rowv = l32 < 16;
        const float Dh = a.D[h];
        uint8_t *sp = sm + OFF_SP;
        uint8_t *gb = sm + OFF_GB;
        uint8_t *yt = sm + OFF_YT;
        float g[P];
        {
            float f0 = 0.f;
            if (Tn > 0) {
                const int64_t i0 = (b * Tn) * H + h;
                f0 = (1.f - a.lam[i0]) * a.dt[i0];
            }
            const int64_t base = (lane_id * N + n) * P;
#pragma unroll
            for (int p = 0; p < P; p += 4) {
                float4 hv = a.h0 ? *reinterpret_cast<const float4 *>(a.h0 + base + p) : make_float4(0, 0, 0, 0);
                float4 uv = a.prevBx0 ? *reinterpret_cast<const float4 *>(a.prevBx0 + base + p)
                                      : make_float4(0, 0, 0, 0);
                g[p] = hv.x + f0 * uv.x;
                g[p + 1] = hv.y + f0 * uv.y;
                g[p + 2] = hv.z + f0 * uv.z;
                g[p + 3] = hv.w + f0 * uv.w;
            }
#pragma unroll
            for (int cc = 0; cc < 8; cc++) {
                uint4 v;
                v.x = pack_bf16(g[8 * cc], g[8 * cc + 1]);
                v.y = pack_bf16(g[8 * cc + 2], g[8 * cc + 3]);
                v.z = pack_bf16(g[8 * cc + 4], g[8 * cc + 5]);
                v.w = pack_bf16(g[8 * cc + 6], g[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(gb + n * 128 + ((cc ^ (n & 7)) << 4)) = v;
            }
            fence_async_smem();
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_STTAKEN));
        }
        const int et = tid - W_EPI0 * 32;
        // one thread waits, the group meets at a named barrier and leaves together
        auto group_wait = [&](int bi, uint32_t parity, int site) -> bool {
            bool fail = false;
            if (et == 0) fail = !wait_bar(bar(bi), parity, abort_flag, a.err, site);
            return !named_bar_or(2, 128, fail);
        };
        bool ok = true;
        for (int c = 0; c < nchunks && ok; c++) {
            const int s = c & 1, k = c >> 1;
            const float *cf = coef0 + s * CF_FLOATS;
            const uint8_t *xr = sm + OFF_STAGE0 + s * STAGE;
            if (!(ok = group_wait(B_CFULL0 + s, k & 1, 20))) break;
            const int L = (int)cf[CF_SCAL + 2];
            const bool unsafe = cf[CF_SCAL + 1] != 0.f;
            // ---- masked scores S' (rows of D1) ----
            if (!(ok = group_wait(B_SFULL, c & 1, 21))) break;
            tc_fence_after();
            {
                const int t = trow;
                const float rt = rowv ? cf[CF_R + t] : 0.f;
                const float c2t = rowv ? cf[CF_C2 + t] : 0.f;
#pragma unroll
                for (int c16 = 0; c16 < Q / 16; c16++) {
                    float v[16];
                    tmem_ld16(tl + COL_D1 + 16 * c16, v);
                    tmem_wait_ld();
                    if (rowv) {
#pragma unroll
                        for (int u = 0; u < 16; u++) {
                            const int s2 = 16 * c16 + u;
                            float m;
                            if (!unsafe)
                                m = s2 < t ? rt * cf[CF_W + s2] : (s2 == t ? rt * cf[CF_GAM + t] : 0.f);
                            else
                                m = s2 < t ? exp2f(c2t - cf[CF_C2 + s2]) * cf[CF_W + s2]
                                           : (s2 == t ? cf[CF_GAM + t] : 0.f);
                            v[u] *= m;
                        }
#pragma unroll
                        for (int hh = 0; hh < 2; hh++) {
                            const int cc = 2 * c16 + hh;
                            uint4 pk;
                            pk.x = pack_bf16(v[8 * hh], v[8 * hh + 1]);
                            pk.y = pack_bf16(v[8 * hh + 2], v[8 * hh + 3]);
                            pk.z = pack_bf16(v[8 * hh + 4], v[8 * hh + 5]);
                            pk.w = pack_bf16(v[8 * hh + 6], v[8 * hh + 7]);
                            *reinterpret_cast<uint4 *>(sp + t * 128 + ((cc ^ (t & 7)) << 4)) = pk;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_STAKEN));
            fence_async_smem();
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_SPFULL));
            // ---- outputs y = D2 + e^{cum_t} D3 + D x ----
            if (et == 0) tma_store_wait_read();   // the previous output tile has been read out
            if (!(ok = group_wait(B_YFULL, c & 1, 22))) break;
            tc_fence_after();
            const float ect = rowv ? cf[CF_EC + trow] : 0.f;
#pragma unroll
            for (int c16 = 0; c16 < P / 16; c16++) {
                float y2[16], y3[16];
                tmem_ld16(tl + COL_D2 + 16 * c16, y2);
                tmem_ld16(tl + COL_D3 + 16 * c16, y3);
                tmem_wait_ld();
                if (rowv) {
                    const int t = trow;
                    uint32_t pk[8];
#pragma unroll
                    for (int hh = 0; hh < 2; hh++) {
                        const int cc = 2 * c16 + hh;   // 16-byte chunk (8 columns)
                        const uint4 xv = *reinterpret_cast<const uint4 *>(xr + t * 128 + ((cc ^ (t & 7)) << 4));
                        const uint32_t *xw = reinterpret_cast<const uint32_t *>(&xv);
#pragma unroll
                        for (int e2 = 0; e2 < 4; e2++) {
                            const float2 xf = unpack_bf16(xw[e2]);
                            const int cidx = 8 * hh + 2 * e2;
                            const float o0 = y2[cidx] + ect * y3[cidx] + Dh * xf.x;
                            const float o1 = y2[cidx + 1] + ect * y3[cidx + 1] + Dh * xf.y;
                            pk[4 * hh + e2] = pack_bf16(o0, o1);
                        }
                        *reinterpret_cast<uint4 *>(yt + t * 128 + ((cc ^ (t & 7)) << 4)) =
                            make_uint4(pk[4 * hh], pk[4 * hh + 1], pk[4 * hh + 2], pk[4 * hh + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_YTAKEN));
            fence_async_smem();
            named_bar(2, 128);
            if (et == 0) {
                tma_store4(&map_y, 0, (int)h, c * Q, (int)b, sbase + OFF_YT);
                mbar_arrive(bar(B_EMPTY0 + s));
            }
            // ---- state: g = e^{cum_end} g + D4 ----
            if (!(ok = group_wait(B_STFULL, c & 1, 23))) break;
            tc_fence_after();
            const float E = cf[CF_SCAL + 0];
#pragma unroll
            for (int c16 = 0; c16 < P / 16; c16++) {
                float d4[16];
                tmem_ld16(tl + COL_D4 + 16 * c16, d4);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; u++) g[16 * c16 + u] = fmaf(E, g[16 * c16 + u], d4[u]);
            }
            tc_fence_before();
#pragma unroll
            for (int cc = 0; cc < 8; cc++) {
                uint4 pk;
                pk.x = pack_bf16(g[8 * cc], g[8 * cc + 1]);
                pk.y = pack_bf16(g[8 * cc + 2], g[8 * cc + 3]);
                pk.z = pack_bf16(g[8 * cc + 4], g[8 * cc + 5]);
                pk.w = pack_bf16(g[8 * cc + 6], g[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(gb + n * 128 + ((cc ^ (n & 7)) << 4)) = pk;
            }
            fence_async_smem();
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_STTAKEN));
            named_bar(2, 128);
            if (et == 0) mbar_arrive(bar(B_CEMPTY0 + s));
            (void)L;
        }
        if (et == 0) tma_store_wait_all();
        // final state: h_{T-1} = g after the last chunk (no lookahead there)
        if (!*abort_flag && a.h_out) {
            float *ho = a.h_out + (lane_id * N + n) * P;
#pragma unroll
            for (int p = 0; p < P; p += 4) *reinterpret_cast<float4 *>(ho + p) = make_float4(g[p], g[p + 1], g[p + 2], g[p + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    // prev_Bx = Bbar_{T-1} x_{T-1}^T (rotated, unscaled B row kept by the rotation warps)
    if (!*abort_flag && a.prevBx_out && warp >= W_EPI0) {
        const int n = tid - W_EPI0 * 32;
        const int c = nchunks - 1, s = c & 1;
        const int L = (int)(Tn - (int64_t)c * Q);
        const uint8_t *xr = sm + OFF_STAGE0 + s * STAGE;
        const int t = L - 1;
        const float bn = blast[n];
        float *uo = a.prevBx_out + (lane_id * N + n) * P;
        for (int cc = 0; cc < 8; cc++) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(xr + t * 128 + ((cc ^ (t & 7)) << 4));
            const uint32_t *xw = reinterpret_cast<const uint32_t *>(&xv);
            float o[8];
            for (int e2 = 0; e2 < 4; e2++) {
                const float2 f = unpack_bf16(xw[e2]);
                o[2 * e2] = bn * f.x;
                o[2 * e2 + 1] = bn * f.y;
            }
            *reinterpret_cast<float4 *>(uo + 8 * cc) = make_float4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<float4 *>(uo + 8 * cc + 4) = make_float4(o[4], o[5], o[6], o[7]);
        }
    }
    if (warp == W_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ---- host side ------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 4-D map over a (Bt, T, H, inner) tensor: dims (inner, H, T, Bt).
static bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int64_t inner,
                     int64_t H, int64_t T, int64_t Bt, uint32_t box_inner, uint32_t box_t, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)Bt};
    cuuint64_t strides[3] = {(cuuint64_t)(inner * esize), (cuuint64_t)(inner * H * esize),
                             (cuuint64_t)(inner * H * T * esize)};
    cuuint32_t box[4] = {box_inner, 1, box_t, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__device__ int g_tc_error;

}  // namespace tc

bool scan_tc_supported(const ScanArgs &a, m3_dtype dt) {
    return dt == M3_BF16 && a.R == 1 && !a.mimo_layout && a.P == tc::P && a.N == tc::N && a.Q == tc::Q &&
           a.T > 0 && a.T <= ((int64_t)1 << 30) && a.Bt <= 65535 && a.H <= 65535;
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t s) {
    using namespace tc;
    CUtensorMap mx, mb, mc, mth, my;
    if (!make_map(&mx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P, a.H, a.T, a.Bt, P, Q, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mb, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, a.H, a.T, a.Bt, N, Q, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mc, a.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, a.H, a.T, a.Bt, N, Q, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mth, a.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, NP2, a.H, a.T, a.Bt, NP2, Q,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&my, a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P, a.H, a.T, a.Bt, P, Q, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    TcArgs t;
    t.dt = a.dt; t.A = a.A; t.lam = a.lam; t.D = a.D;
    t.h0 = a.h0; t.prevBx0 = a.prevBx0; t.angle0 = a.angle0;
    t.nrm = a.nrm;
    t.h_out = a.h_out; t.prevBx_out = a.prevBx_out; t.angle_out = a.angle_out;
    t.Bt = a.Bt; t.T = a.T; t.H = a.H;
    int *err = nullptr;
    cudaGetSymbolAddress(reinterpret_cast<void **>(&err), g_tc_error);
    t.err = err;
    cudaFuncSetAttribute(k_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    k_scan_tc<<<(unsigned)(a.Bt * a.H), THREADS, SMEM_BYTES, s>>>(mx, mb, mc, mth, my, t);
    count_launch();
    return cudaGetLastError();
}

int scan_tc_error_and_clear(cudaStream_t s) {
    int *err = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&err), tc::g_tc_error) != cudaSuccess) return -1;
    int v = 0;
    if (cudaMemcpyAsync(&v, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return -1;
    if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
    if (v) {
        const int zero = 0;
        if (cudaMemcpyAsync(err, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess) return -1;
        if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace m3
