// k_scan_tc.cu -- chunked forward of the Mamba-3 scan, SISO and rank-R MIMO,
// on the sm_100a tensor cores (bf16 inputs, headdim 64, dState 128).
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
// MIMO (rank R, TorchMamba README "Math notes": rank-R update on a shared
// (N,P) state; App. C per-head expand/contract vectors) is the same chunked
// form with R rows (t, r) per token: X_{t,r} = W_x[r] x_t, the mask depends on
// the tokens only, the state update sums over all rows, and
// y_t = sum_r W_y[r] Y_{t,r} + D x_t.  A chunk always holds 64 rows, i.e.
// 64 / R tokens, so the UMMA shapes below are the same for every R.
//
// One CTA owns one (b, h) lane -- or one segment of it, see below -- and
// walks its chunks in order.  Per chunk four UMMAs (tcgen05.mma kind::f16,
// bf16 operands in shared memory, fp32 accumulators in tensor memory):
//   D1 = Cbar . Bbar^T            scores            M=64  N=64  K=128
//   D3 = Cbar . g_in              inter-chunk term  M=64  N=64  K=128
//   D2 = S' . X                   intra-chunk term  M=64  N=64  K=64
//   D4 = Bbar^T . Xw              chunk state       M=128 N=64  K=64
// With e_s = e^{cum_end - cum_s}, Xw holds e_s w_s x_s, so D4 is the chunk's
// state contribution directly, and the decay mask is split into a row factor
// r_t = e^{cum_t - cum_end} and a column factor e_s w_s (gamma_t on the
// diagonal, zero above it), applied to D1 in the epilogue.  When a chunk's
// log-decay range exceeds 60 the two factors could leave the fp32 range; such
// a chunk's scores instead get the exact factor e^{cum_t - cum_s} w_s one by
// one.
//
// Long sequences over few lanes are cut into segments of whole chunks: a
// state-only pass computes every segment's end state from a zero start in
// its own angle frame, a small combine kernel chains the segments, and the
// full pass then runs all segments in parallel from their entering states.
//
// Warp roles (20 warps): 0 the X operands (Xw, and the rank-expanded X_r for
// MIMO), 1 MMA issuer (and TMEM owner), 2 per-token coefficients, 3-10
// rotation (QkNorm, bias, RoPE; each thread 4 pairs x 4 tokens with 16-byte
// shared-memory accesses), 11-18 epilogue (two warps per TMEM lane quarter,
// each owning 32 of the 64 columns: masked scores, fp32 state in registers,
// outputs), 19 TMA producer.  Inputs stream
// through two rings: B, C, theta (released once rotated) and x (released
// once the outputs are written).  Every wait is bounded: past ~1 s the kernel
// records an error, stops issuing work, drains what it has in flight and
// returns.
#include <cuda.h>

#include "m3_internal.cuh"

namespace m3 {
namespace tc {

template <bool V> struct BoolC { static constexpr bool value = V; };

constexpr int Q = 64, P = 64, N = 128, NP2 = 64;
constexpr int NWARPS = 20, THREADS = NWARPS * 32;
// The X-operand warp is warp 0 and the TMA producer warp 19: measured 2.4 %
// faster MIMO rank 4 (whose X operands are twice the work) than the other way
// round, the same for SISO.
constexpr int W_XB = 0, W_MMA = 1, W_COEF = 2, W_PREP0 = 3, NPREP = 8, W_EPI0 = 11, W_TMA = 19;
constexpr int PREP_THREADS = NPREP * 32;          // 256
constexpr int EPI_THREADS = 256;                  // two warps per TMEM lane quarter
constexpr int EPI_WARPS = EPI_THREADS / 32;

// ---- shared-memory map (bytes from a 1024-aligned base) ------------------
// Rank R: a chunk holds QT = Q / R tokens and Q rows (token, rank) of B and C;
// the x, theta and output tiles have QT rows, and MIMO (R > 1) adds the
// rank-expanded X_r = W_x[r] * x, the W_x / W_y vectors and R rows of the
// last token's rotated B.
constexpr int NB = 2, NX = 3, NC = 4;             // ring depths: B/C, x, coefficients
constexpr int SZ_BC = Q * N * 2;                  // 16 KB, bf16, row-major (TMA)
constexpr int SZ_SP = Q * Q * 2, SZ_GB = N * P * 2;
// per-chunk coefficient buffer (a ring of NC), floats; per token of the chunk
constexpr int CF_W = 0, CF_GAM = Q, CF_R = 2 * Q, CF_EC = 3 * Q, CF_XS = 4 * Q, CF_C2 = 5 * Q, CF_DT = 6 * Q,
              CF_WM = 7 * Q, CF_SCAL = 8 * Q, CF_FLOATS = 8 * Q + 8;
template <int R>
struct Lay {
    static constexpr int QT = Q / R;
    static constexpr int NXR = (R == 2) ? 2 : NX;             // x ring depth (rank 2: shared memory is full)
    static constexpr int SZ_X = QT * P * 2;                   // bf16, 128B-swizzled (TMA)
    static constexpr int SZ_BCT = 2 * SZ_BC;                  // one B/C stage
    static constexpr int OFF_BCT = 0;                         // NB x [B | C]
    static constexpr int OFF_X = OFF_BCT + NB * SZ_BCT;       // NX x [QT][P]
    static constexpr int OFF_BB = ((OFF_X + NXR * SZ_X + 1023) / 1024) * 1024;   // 2 x [2 atoms][Q rows][64]
    static constexpr int OFF_CB = OFF_BB + 2 * Q * N * 2;    // 2 x [2 atoms][Q rows][64] bf16, SW128
    static constexpr int OFF_SP = OFF_CB + 2 * Q * N * 2;     // [Q][Q] bf16, SW128
    static constexpr int OFF_XW = OFF_SP + SZ_SP;             // 2 x [Q rows][P] bf16, SW128
    static constexpr int OFF_XR = OFF_XW + 2 * Q * P * 2;     // 2 x [Q rows][P] bf16, SW128 (R > 1)
    static constexpr int OFF_GB = OFF_XR + (R > 1 ? 2 * Q * P * 2 : 0);   // 2 x [N][P] bf16, SW128
    static constexpr int OFF_COEF = OFF_GB + 2 * SZ_GB;
    static constexpr int OFF_BLAST = OFF_COEF + NC * CF_FLOATS * 4;  // fp32 [R][N]
    static constexpr int OFF_WXY = OFF_BLAST + R * N * 4;            // fp32 [2][R][P] (R > 1)
    static constexpr int OFF_PHIC = OFF_WXY + (R > 1 ? 2 * R * P * 4 : 0);  // fp32 [NP2]
    static constexpr int OFF_PART = OFF_PHIC + NP2 * 4;       // fp32 [8][NP2] per-warp angle sums
    static constexpr int OFF_INV = OFF_PART + 8 * NP2 * 4;    // fp32 [2][Q] QkNorm inverse RMS
    static constexpr int OFF_BAR = OFF_INV + 2 * Q * 4;       // mbarriers
};

// barrier indices
enum {
    B_BFULL = 0,                    // NB: B/C/theta stage loaded (TMA)
    B_BEMPTY = B_BFULL + NB,        // NB: stage rotated
    B_XFULL = B_BEMPTY + NB,        // NX: x tile loaded (TMA)
    B_XEMPTY = B_XFULL + NX,        // NX: Xw built, intra UMMA done, outputs written
    B_CFULL = B_XEMPTY + NX,        // NC: coefficients ready
    B_CEMPTY = B_CFULL + NC,        // NC: coefficients consumed
    B_OPSREADY = B_CEMPTY + NC,     // 2: rotated operands and Xw written (double-buffered)
    B_OPSFREE = B_OPSREADY + 2,     // 2: the UMMAs reading them are done
    B_SFULL = B_OPSFREE + 2,
    B_STAKEN, B_SPFULL,             // scores in TMEM / read / masked scores written
    B_YFULL,                        // output accumulators done
    B_YTAKEN,                       // 2: inter-chunk accumulator (double-buffered) read
    B_STFULL = B_YTAKEN + 2,        // chunk state done
    B_STTAKEN,                      // chunk state folded into the state
    B_DRAIN,
    NBAR
};
template <int R>
constexpr int smem_bytes() { return Lay<R>::OFF_BAR + NBAR * 8 + 16 + 1024; }   // + misc + alignment slack
static_assert(smem_bytes<1>() <= 227 * 1024 && smem_bytes<2>() <= 227 * 1024 && smem_bytes<4>() <= 227 * 1024,
              "shared memory budget");

// D3 is double-buffered (chunk c uses COL_D3 + (c & 1) * D3_STRIDE), so the
// inter-chunk UMMA of chunk c does not wait for the outputs of chunk c-1
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_D1 = 0, COL_D2 = 64, COL_D3 = 128, COL_D4 = 192, D3_STRIDE = 128;

struct TcArgs {
    void *y;               // (Bt, T, H, P) bf16
    const float *theta;    // (Bt, T, H, K) fp32
    const float *dt, *A, *lam, *D;
    const float *Wx, *Wy;  // MIMO expand / contract vectors (H, R, P), NULL = ones
    const float *h0, *prevBx0, *angle0;
    NormArgs nrm;
    float *h_out, *prevBx_out, *angle_out;
    int64_t Bt, T, H;
    int64_t G;         // B/C groups: head h reads group h / (H / G)
    int K;             // rotated pairs (a multiple of 4, <= N/2); pairs >= K pass through
    int64_t seg_len;   // tokens per segment (a multiple of Q); one segment covers the whole sequence
    int nseg;          // segments per lane
    float *ws;         // segment slots (nseg > 1)
    int *err;
};

// Workspace slot of one (lane, segment j < nseg-1), in floats:
//   [0, N*P)        after the state-only pass: the segment's end state from a
//                   zero start, in the segment's own angle frame; after the
//                   combine pass: the state entering segment j+1
//   [N*P, +N/2)     angle increment over segment j
//   [+N/2, +N/2)    angle entering segment j+1
//   [N*P + N]       product of alpha over segment j
constexpr int SLOT_G = 0, SLOT_PHIL = N * P, SLOT_PHIN = N * P + NP2, SLOT_E = N * P + N;
constexpr int SLOT_FLOATS = N * P + N + 4;

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
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(10000000u)   // suspend up to 10 ms instead of spinning
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_try_spin(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

constexpr long long WAIT_LIMIT_CYCLES = 2000000000LL;  // ~1 s at 1.9 GHz

// Bounded wait without the suspend hint (for the single MMA-issuing thread).
// The first probe is inline; the polling loop is one out-of-line copy shared
// by every call site, which keeps the hot loops of the kernel small.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                           int site, bool spin) {
    const long long t0 = clock64();
    while (true) {
        if (spin ? mbar_try_spin(bar, parity) : mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
            *abort_flag = 1;
            atomicCAS(err, 0, site);
            return false;
        }
    }
}
__device__ __forceinline__ bool wait_bar_spin(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                              int site) {
    return mbar_try_spin(bar, parity) || wait_bar_slow(bar, parity, abort_flag, err, site, true);
}
// Bounded waits taken by every lane of a converged warp, with one warp-wide
// outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                          int site);
__device__ __forceinline__ bool warp_wait_spin(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                               int site) {
    const bool ok = wait_bar_spin(bar, parity, abort_flag, err, site);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait on an mbarrier phase.  Returns false when the kernel is
// aborting (this wait timed out, or another thread's did).  Every role polls
// without the suspend-time hint: measured on the default, MIMO and long
// workloads, the hinted form woke waiting warps later (2-5 % slower calls).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                         int site) {
    return mbar_try_spin(bar, parity) || wait_bar_slow(bar, parity, abort_flag, err, site, true);
}
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *err,
                                          int site) {
    const bool ok = wait_bar(bar, parity, abort_flag, err, site);
    return __all_sync(0xffffffffu, ok);
}

// One lane of a converged warp (elect.sync): the lane that issues a UMMA, a
// commit or a TMA copy, while the whole warp computes the (warp-uniform)
// operands.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n .reg .b32 rx;\n .reg .pred px;\n elect.sync rx|px, 0xffffffff;\n selp.b32 %0, 1, 0, px;\n}"
        : "=r"(pred));
    return pred != 0;
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
__device__ __forceinline__ void tma_load5(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3, int c4,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], "
        "[%7];" ::"r"(dst),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_prefetch5(const CUtensorMap *map, int c0, int c1, int c2, int c3, int c4) {
    asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global [%0, {%1, %2, %3, %4, %5}];" ::"l"(map), "r"(c0),
                 "r"(c1), "r"(c2), "r"(c3), "r"(c4)
                 : "memory");
}
// Pull a box of the tensor into L2 ahead of its load (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch4(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global [%0, {%1, %2, %3, %4}];" ::"l"(map), "r"(c0), "r"(c1),
                 "r"(c2), "r"(c3)
                 : "memory");
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
// 32 fp32 columns of 16 TMEM lanes (the rows of an M=64 accumulator in this
// warp's lane quarter), spread over the 32 threads: thread t gets, for each
// group i of 8 columns, v[4i], v[4i+1] = (lane t/4, columns 8i + 2(t%4) + 0, 1)
// and v[4i+2], v[4i+3] = (lane t/4 + 8, the same columns).
__device__ __forceinline__ void tmem_ld16x256b_x4(uint32_t taddr, float *v) {
    uint32_t r[16];
    __syncwarp();
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}
// The same for 16 columns (two groups of 8).
__device__ __forceinline__ void tmem_ld16x256b_x2(uint32_t taddr, float *v) {
    uint32_t r[8];
    __syncwarp();
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = __uint_as_float(r[i]);
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
constexpr float INV_2PI = 0.15915494309189535f, TWO_PI_HI = 6.28125f, TWO_PI_LO = 1.9353071795864769e-3f;
__device__ __forceinline__ float reduce_2pi(float x) {
    const float k = rintf(x * INV_2PI);
    return fmaf(-k, TWO_PI_LO, fmaf(-k, TWO_PI_HI, x));
}
__device__ __forceinline__ void sincos_rr(float x, float *s, float *c) { __sincosf(reduce_2pi(x), s, c); }

// SO (state only): the first pass over all but the last segment of each lane;
// it loads x, B, theta (no C), runs only the chunk-state UMMA, starts from a
// zero state in the segment's own angle frame and writes the segment's end
// state, angle increment and decay product to its workspace slot.
template <bool SO, int R>
__global__ void __launch_bounds__(THREADS, 1)
    k_scan_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
              const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_th, TcArgs a) {
    using L = Lay<R>;
    constexpr int QT = L::QT;                          // tokens per chunk
    constexpr int TPT = QT / 16;                       // tokens per rotation thread
    constexpr int OFF_MISC = L::OFF_BAR + NBAR * 8;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, l32 = tid & 31;
    const int nsb = SO ? a.nseg - 1 : a.nseg;          // CTAs per lane in this pass
    const int64_t lane_id = blockIdx.x / nsb, b = lane_id / a.H, h = lane_id % a.H;
    const int hg = (int)(h / (a.H / a.G));                // B/C group of this head
    const int seg = blockIdx.x % nsb;
    const int64_t Tn = a.T, H = a.H;
    const int64_t t_beg = (int64_t)seg * a.seg_len;
    const int64_t t_end = (t_beg + a.seg_len < Tn) ? t_beg + a.seg_len : Tn;
    const int nchunks = (int)((t_end - t_beg + QT - 1) / QT);
    const bool last_seg = SO ? false : (seg == a.nseg - 1);
    float *slot_in = (!SO && seg > 0) ? a.ws + ((size_t)lane_id * (a.nseg - 1) + (seg - 1)) * SLOT_FLOATS : nullptr;
    float *slot_out = SO ? a.ws + ((size_t)lane_id * (a.nseg - 1) + seg) * SLOT_FLOATS : nullptr;
    auto bar = [&](int i) { return sbase + L::OFF_BAR + 8 * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    float *coef0 = reinterpret_cast<float *>(sm + L::OFF_COEF);
    float *blast = reinterpret_cast<float *>(sm + L::OFF_BLAST);
    float *wxs = reinterpret_cast<float *>(sm + L::OFF_WXY);            // [R][P] (R > 1)
    float *wys = wxs + R * P;                                            // [R][P] (R > 1)
    float *phic = reinterpret_cast<float *>(sm + L::OFF_PHIC);
    float *part = reinterpret_cast<float *>(sm + L::OFF_PART);
    float *inv = reinterpret_cast<float *>(sm + L::OFF_INV);

    if (tid == 0) {
        for (int i = 0; i < NB; i++) {
            mbar_init(bar(B_BFULL + i), 1);
            mbar_init(bar(B_BEMPTY + i), 1);
        }
        // x tiles are released by the X-operand warp, the intra UMMA and (MIMO)
        // each of the eight output-writing warps (state-only pass: the
        // X-operand warp alone); coefficients by the rotation group, the X-operand warp
        // and each epilogue warp; a chunk's operands are ready once both the
        // rotation group and the X-operand warp have written theirs
        for (int i = 0; i < L::NXR; i++) {
            mbar_init(bar(B_XFULL + i), 1);
            mbar_init(bar(B_XEMPTY + i), SO ? 1 : (R == 1 ? 2 : 2 + EPI_WARPS));
        }
        for (int i = 0; i < NC; i++) {
            mbar_init(bar(B_CFULL + i), 1);
            mbar_init(bar(B_CEMPTY + i), 2 + EPI_WARPS);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(bar(B_OPSREADY + i), 2);
            mbar_init(bar(B_OPSFREE + i), 1);
        }
        mbar_init(bar(B_SFULL), 1);
        mbar_init(bar(B_STAKEN), 8);
        mbar_init(bar(B_SPFULL), 8);
        mbar_init(bar(B_YFULL), 1);
        mbar_init(bar(B_YTAKEN), 8);
        mbar_init(bar(B_YTAKEN + 1), 8);
        mbar_init(bar(B_STFULL), 1);
        mbar_init(bar(B_STTAKEN), 8);
        mbar_init(bar(B_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_x) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_b) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_c) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&map_th) : "memory");
    }
    if (warp == W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (R > 1) {
        for (int k = tid; k < R * P; k += THREADS) {
            wxs[k] = a.Wx ? a.Wx[h * R * P + k] : 1.f;
            wys[k] = a.Wy ? a.Wy[h * R * P + k] : 1.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // ------------------------------------------------------------ producer
        // converged warp, warp-uniform coordinates, one elected lane issues
        {
            // B and C of a chunk: rows (token, rank) of this head's group -- a
            // 4-D box (N, G, T, Bt) for SISO, a 5-D box (N, R, G, T, Bt) for MIMO
            auto load_bc = [&](uint32_t dst, const CUtensorMap *m, int t0, uint32_t fb) {
                if (R == 1) tma_load4(dst, m, 0, hg, t0, (int)b, fb);
                else tma_load5(dst, m, 0, 0, hg, t0, (int)b, fb);
            };
            auto prefetch_bc = [&](const CUtensorMap *m, int t0) {
                if (R == 1) tma_prefetch4(m, 0, hg, t0, (int)b);
                else tma_prefetch5(m, 0, 0, hg, t0, (int)b);
            };
            // L2 prefetch runs PFD chunks ahead of the shared-memory rings, so
            // a load issued when a stage frees up finds its data in L2
            constexpr int PFD = 3;
            auto prefetch = [&](int c) {
                if (c >= nchunks) return;
                const int t0 = (int)(t_beg + (int64_t)c * QT);
                prefetch_bc(&map_b, t0);
                if (!SO) prefetch_bc(&map_c, t0);
                tma_prefetch4(&map_th, 0, (int)h, t0, (int)b);
                tma_prefetch4(&map_x, 0, (int)h, t0, (int)b);
            };
            int issued = 0;
            for (int c = 0; c < nchunks; c++) {
                const int sb = c % NB, kb = c / NB, sx = c % L::NXR, kx = c / L::NXR;
                const int t0 = (int)(t_beg + (int64_t)c * QT);
                if (kb > 0 && !warp_wait(bar(B_BEMPTY + sb), (kb - 1) & 1, abort_flag, a.err, 1)) break;
                const uint32_t st = sbase + L::OFF_BCT + sb * L::SZ_BCT;
                const uint32_t fb = bar(B_BFULL + sb);
                if (elect_one()) {
                    mbar_expect_tx(fb, SO ? SZ_BC : L::SZ_BCT);
                    load_bc(st, &map_b, t0, fb);
                    if (!SO) load_bc(st + SZ_BC, &map_c, t0, fb);
                }
                __syncwarp();
                if (kx > 0 && !warp_wait(bar(B_XEMPTY + sx), (kx - 1) & 1, abort_flag, a.err, 2)) break;
                const uint32_t xb = bar(B_XFULL + sx);
                if (elect_one()) {
                    mbar_expect_tx(xb, L::SZ_X);
                    tma_load4(sbase + L::OFF_X + sx * L::SZ_X, &map_x, 0, (int)h, t0, (int)b, xb);
                    // the L2 prefetches go out after this chunk's loads: at the
                    // start every CTA's first chunk then comes before the
                    // look-ahead traffic of all of them
                    if (c == 0)
                        for (int k = 1; k <= PFD; k++) prefetch(k);
                    else
                        prefetch(c + PFD);
                }
                __syncwarp();
                issued = c + 1;
            }
            // never leave loads in flight into shared memory at exit
            for (int c = (issued > L::NXR ? issued - L::NXR : 0); c < issued; c++) {
                const long long t0 = clock64();
                while (!mbar_try(bar(B_XFULL + c % L::NXR), (c / L::NXR) & 1) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
                }
            }
            for (int c = (issued > NB ? issued - NB : 0); c < issued; c++) {
                const long long t0 = clock64();
                while (!mbar_try(bar(B_BFULL + c % NB), (c / NB) & 1) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
                }
            }
        }
    } else if (warp == W_COEF) {
        // --------------------------------------------------------- coefficients
        const float L2E = 1.4426950408889634f;
        const float A2 = a.A[h] * L2E;
        const float UNSAFE2 = 60.f * L2E;
        for (int c = 0; c < nchunks; c++) {
            const int s = c % NC, k = c / NC;
            // fetch this chunk's dt and lam before waiting for the buffer
            const int64_t t0 = t_beg + (int64_t)c * QT;
            const int Lc = (int)((t_end - t0) < QT ? (t_end - t0) : QT);
            float dl[2], lm[2], dn[2], ln[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i = l32 + 32 * u;
                dl[u] = lm[u] = dn[u] = 0.f;
                ln[u] = 1.f;
                if (i < Lc) {
                    const int64_t bt = (b * Tn + t0 + i) * H + h;
                    dl[u] = a.dt[bt];
                    lm[u] = a.lam[bt];
                    if (t0 + i + 1 < Tn) {
                        dn[u] = a.dt[bt + H];
                        ln[u] = a.lam[bt + H];
                    }
                }
            }
            int ok = 1;
            if (l32 == 0 && k > 0) ok = wait_bar(bar(B_CEMPTY + s), (k - 1) & 1, abort_flag, a.err, 3);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            float *cf = coef0 + s * CF_FLOATS;
            float la[2], wv[2], gv[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
                gv[u] = lm[u] * dl[u];
                wv[u] = gv[u] + (1.f - ln[u]) * dn[u];
                la[u] = dl[u] * A2;
            }
            // inclusive scan of log2(alpha) over the chunk's tokens
#pragma unroll
            for (int u = 0; u < 2; u++)
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, la[u], o);
                    if (l32 >= o) la[u] += v;
                }
            la[1] += __shfl_sync(0xffffffffu, la[0], 31);
            const float cend = __shfl_sync(0xffffffffu, (Lc - 1) < 32 ? la[0] : la[1], (Lc - 1) & 31);
            float dev = 0.f;
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i = l32 + 32 * u;
                if (i >= Lc) la[u] = cend;
                dev = fmaxf(dev, fabsf(la[u] - cend));
            }
            const bool unsafe = __any_sync(0xffffffffu, dev > UNSAFE2);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int i = l32 + 32 * u;
                if (i < QT) {
                    // e_s = e^{cum_end - cum_s} goes into the X operand of the
                    // chunk-state UMMA (Xw = e_s w_s x_s) and into the mask's
                    // column factor; the mask is r_t * (e_s w_s), or ones when the
                    // chunk takes the exact path (the scores then get
                    // e^{cum_t - cum_s} w_s one by one)
                    const float ew = exp2f(cend - la[u]) * wv[u];
                    cf[CF_W + i] = wv[u];
                    cf[CF_WM + i] = unsafe ? 1.f : ew;
                    cf[CF_GAM + i] = gv[u];
                    cf[CF_R + i] = unsafe ? 1.f : exp2f(la[u] - cend);
                    cf[CF_EC + i] = exp2f(la[u]);
                    cf[CF_XS + i] = ew;
                    cf[CF_C2 + i] = la[u];
                    cf[CF_DT + i] = dl[u];
                }
            }
            if (l32 == 0) {
                cf[CF_SCAL + 0] = exp2f(cend);
                cf[CF_SCAL + 1] = unsafe ? 1.f : 0.f;
                cf[CF_SCAL + 2] = (float)Lc;
            }
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_CFULL + s));
        }
    } else if (warp >= W_PREP0 && warp < W_PREP0 + NPREP) {
        // --------------- QkNorm + bias + RoPE rotation, then the X operands
        // thread (j4, tg): pairs 4*j4 .. 4*j4+3 (elements 8*j4 .. 8*j4+7, one
        // 16-byte chunk) of tokens TPT*tg .. TPT*tg+TPT-1, all ranks of each
        const int pt = tid - W_PREP0 * 32;         // 0..255
        const int j4 = pt & 15, tg = pt >> 4;
        const NormArgs nr = a.nrm;
        const bool has_norm = nr.wB || nr.wC;
        const bool has_bias = nr.biasB || nr.biasC;
        const uint32_t atom = (uint32_t)(j4 >> 3) * (Q * 128);
        const int chk = j4 & 7;                    // 16-byte chunk within the 128-byte atom row
        const int i0 = tg * TPT;
        if (pt < NP2) {
            // the angle entering the first chunk (read after the first named barrier
            // of the chunk loop); state-only: the segment's own frame, zero
            float p0 = 0.f;
            if (!SO)
                p0 = slot_in ? slot_in[SLOT_PHIN + pt]
                             : ((a.angle0 && pt < a.K) ? a.angle0[lane_id * a.K + pt] : 0.f);
            phic[pt] = p0;
        }
        // theta of my tokens comes straight from global memory into registers,
        // one chunk ahead (the producer has already pulled it into L2).  Pairs
        // from K on take theta = 0: their angle stays 0 and they pass through.
        const float4 *thg = reinterpret_cast<const float4 *>(a.theta);
        const int K4 = a.K / 4;
        const bool turns = j4 < K4;
        float4 thv[TPT];
        auto load_theta = [&](int c) {
            const int64_t t0 = t_beg + (int64_t)c * QT;
#pragma unroll
            for (int u = 0; u < TPT; u++) {
                const int64_t t = t0 + i0 + u;
                thv[u] = (c < nchunks && t < t_end && turns) ? thg[((b * Tn + t) * H + h) * K4 + j4]
                                                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        // QkNorm gain and BC-bias of pair q of one raw row (QkNorm / bias variant)
        auto norm_bias = [&](int row, int r, int q, float2 &bv, float2 &cv) {
            const int e0 = 8 * j4 + 2 * q;
            const int64_t bo = (h * R + r) * N + e0;
            if (nr.wB) { const float ib = inv[row]; bv.x *= ib * nr.wB[e0]; bv.y *= ib * nr.wB[e0 + 1]; }
            if (nr.wC) { const float ic = inv[Q + row]; cv.x *= ic * nr.wC[e0]; cv.y *= ic * nr.wC[e0 + 1]; }
            if (nr.biasB) { bv.x += nr.biasB[bo]; bv.y += nr.biasB[bo + 1]; }
            if (nr.biasC) { cv.x += nr.biasC[bo]; cv.y += nr.biasC[bo + 1]; }
        };
        load_theta(0);
        for (int c = 0; c < nchunks; c++) {
            const int sb = c % NB, kb = c / NB, scf = c % NC, kc = c / NC;
            const int ob = c & 1;                  // operand buffer
            bool fail = false;
            if (pt == 0) {
                fail = !(wait_bar(bar(B_BFULL + sb), kb & 1, abort_flag, a.err, 4) &&
                         wait_bar(bar(B_CFULL + scf), kc & 1, abort_flag, a.err, 6) &&
                         (c < 2 || wait_bar(bar(B_OPSFREE + ob), ((c >> 1) - 1) & 1, abort_flag, a.err, 7)));
            }
            if (named_bar_or(1, PREP_THREADS, fail)) break;
            uint8_t *bbar = sm + L::OFF_BB + ob * (Q * N * 2);
            uint8_t *cb = sm + L::OFF_CB + ob * (Q * N * 2);
            const float *cf = coef0 + scf * CF_FLOATS;
            const uint8_t *stg = sm + L::OFF_BCT + sb * L::SZ_BCT;
            const uint4 *braw = reinterpret_cast<const uint4 *>(stg);
            const uint4 *craw = reinterpret_cast<const uint4 *>(stg + SZ_BC);
            const int Lc = (int)cf[CF_SCAL + 2];
            if (has_norm) {
                // inverse RMS of each B and C row of the chunk: one warp per row
                const int wp = pt >> 5;
                const uint32_t *b32 = reinterpret_cast<const uint32_t *>(braw);
                const uint32_t *c32 = reinterpret_cast<const uint32_t *>(craw);
                for (int r = wp; r < 2 * Q; r += NPREP) {
                    const int i = r & (Q - 1);
                    const uint32_t *raw = (r < Q) ? b32 : c32;
                    float ss = 0.f;
                    for (int qq = l32; qq < NP2; qq += 32) {
                        const float2 f = unpack_bf16(raw[i * NP2 + qq]);
                        ss += f.x * f.x + f.y * f.y;
                    }
                    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    if (l32 == 0) inv[r] = rsqrtf(ss / N + nr.eps);
                }
            }
            // pass 1: angle increments of my token group, then the angle entering
            // it: the chunk's entering angle + the earlier warps' sums + (second
            // token group of a warp) the first group's sum
            float dph[TPT][4];
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            float amax = 0.f;                      // bound on my angle's drift inside the chunk
#pragma unroll
            for (int u = 0; u < TPT; u++) {
                const float d = cf[CF_DT + i0 + u];
                const float4 t4 = thv[u];
                dph[u][0] = d * t4.x;
                dph[u][1] = d * t4.y;
                dph[u][2] = d * t4.z;
                dph[u][3] = d * t4.w;
#pragma unroll
                for (int q = 0; q < 4; q++) acc[q] += dph[u][q];
                amax += fmaxf(fmaxf(fabsf(dph[u][0]), fabsf(dph[u][1])), fmaxf(fabsf(dph[u][2]), fabsf(dph[u][3])));
            }
            const int wp = pt >> 5;
            float first[4];                        // the warp's first token group's sums
#pragma unroll
            for (int q = 0; q < 4; q++) first[q] = __shfl_sync(0xffffffffu, acc[q], l32 & 15);
            if (l32 >= 16)
                *reinterpret_cast<float4 *>(part + wp * NP2 + 4 * j4) =
                    make_float4(first[0] + acc[0], first[1] + acc[1], first[2] + acc[2], first[3] + acc[3]);
            named_bar(1, PREP_THREADS);
            float phi[4];
            {
                const float4 p0 = *reinterpret_cast<const float4 *>(phic + 4 * j4);
                phi[0] = p0.x; phi[1] = p0.y; phi[2] = p0.z; phi[3] = p0.w;
#pragma unroll
                for (int w2 = 0; w2 < NPREP - 1; w2++) {
                    if (w2 < wp) {
                        const float4 pg = *reinterpret_cast<const float4 *>(part + w2 * NP2 + 4 * j4);
                        phi[0] += pg.x; phi[1] += pg.y; phi[2] += pg.z; phi[3] += pg.w;
                    }
                }
                if (l32 >= 16) {
#pragma unroll
                    for (int q = 0; q < 4; q++) phi[q] += first[q];
                }
            }
            // sin/cos of a small angle need no range reduction per token: reduce
            // the entering angle once and advance the reduced copy, unless some
            // increment is large (then every token reduces its own angle)
            const bool fast = !__any_sync(0xffffffffu, amax > 256.f);
            float phr[4];
#pragma unroll
            for (int q = 0; q < 4; q++) phr[q] = reduce_2pi(phi[q]);
            // pass 2: rotate my tokens (the same angles for every rank).  In the
            // plain variant the body has no branches: rows past the sequence end
            // were zero-filled by the TMA load (a chunk ends inside its segment
            // only at the sequence end), so they rotate to zeros.  The QkNorm /
            // bias variant is a separate copy that skips those rows (a bias or a
            // zero-row norm would make them non-zero there).
            const float phi_in[4] = {phi[0], phi[1], phi[2], phi[3]};   // angle entering my tokens
            auto rotate_tokens = [&](auto generic, auto fast_sc) {
                constexpr bool G = decltype(generic)::value, F = decltype(fast_sc)::value;
#pragma unroll
                for (int u = 0; u < TPT; u++) {
                    const int i = i0 + u;
                    float sn[4], cs[4];
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        if (F) {
                            phr[q] += dph[u][q];
                            __sincosf(phr[q], &sn[q], &cs[q]);
                        } else {
                            phi[q] += dph[u][q];
                            sincos_rr(phi[q], &sn[q], &cs[q]);
                        }
                    }
#pragma unroll
                    for (int r = 0; r < R; r++) {
                        const int row = i * R + r;
                        uint4 ob = make_uint4(0u, 0u, 0u, 0u), oc = make_uint4(0u, 0u, 0u, 0u);
                        if (!G || i < Lc) {
                            const uint4 rb = braw[row * 16 + j4];
                            const uint4 rc = SO ? make_uint4(0u, 0u, 0u, 0u) : craw[row * 16 + j4];
                            const uint32_t rbw[4] = {rb.x, rb.y, rb.z, rb.w}, rcw[4] = {rc.x, rc.y, rc.z, rc.w};
                            uint32_t pbw[4], pcw[4];
#pragma unroll
                            for (int q = 0; q < 4; q++) {
                                float2 bv = unpack_bf16(rbw[q]), cv = unpack_bf16(rcw[q]);
                                if (G) norm_bias(row, r, q, bv, cv);
                                pbw[q] = pack_bf16(cs[q] * bv.x - sn[q] * bv.y, sn[q] * bv.x + cs[q] * bv.y);
                                pcw[q] = SO ? 0u : pack_bf16(cs[q] * cv.x - sn[q] * cv.y, sn[q] * cv.x + cs[q] * cv.y);
                            }
                            ob = make_uint4(pbw[0], pbw[1], pbw[2], pbw[3]);
                            oc = make_uint4(pcw[0], pcw[1], pcw[2], pcw[3]);
                        }
                        const uint32_t off = atom + (uint32_t)(row * 128 + ((chk ^ (row & 7)) << 4));
                        *reinterpret_cast<uint4 *>(bbar + off) = ob;
                        if (!SO) *reinterpret_cast<uint4 *>(cb + off) = oc;
                    }
                }
            };
            if (has_norm || has_bias) {
                rotate_tokens(BoolC<true>{}, BoolC<false>{});
            } else if (fast) {
                rotate_tokens(BoolC<false>{}, BoolC<true>{});
#pragma unroll
                for (int q = 0; q < 4; q++) phi[q] += acc[q];   // the exact angle after my tokens
            } else {
                rotate_tokens(BoolC<false>{}, BoolC<false>{});
            }
            if (last_seg && c == nchunks - 1) {
                // the sequence's last token: its rotated B rows in fp32, for
                // prev_Bx (once per lane, off the hot loop)
                const int ul = Lc - 1 - i0;
                if (ul >= 0 && ul < TPT) {
                    float sn[4], cs[4];
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        float ang = phi_in[q];
#pragma unroll
                        for (int u = 0; u < TPT; u++)
                            if (u <= ul) ang += dph[u][q];
                        sincos_rr(ang, &sn[q], &cs[q]);
                    }
                    for (int r = 0; r < R; r++) {
                        const int row = (i0 + ul) * R + r;
                        const uint4 rb = braw[row * 16 + j4];
                        const uint32_t rbw[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
                        for (int q = 0; q < 4; q++) {
                            float2 bv = unpack_bf16(rbw[q]), cv = make_float2(0.f, 0.f);
                            if (has_norm || has_bias) norm_bias(row, r, q, bv, cv);
                            blast[r * N + 8 * j4 + 2 * q] = cs[q] * bv.x - sn[q] * bv.y;
                            blast[r * N + 8 * j4 + 2 * q + 1] = sn[q] * bv.x + cs[q] * bv.y;
                        }
                    }
                }
            }
            load_theta(c + 1);                     // in flight while the X operands are built
            fence_async_smem();
            named_bar(1, PREP_THREADS);
            if (tg == 15) {
                // the last token group ends at the chunk's last token
                *reinterpret_cast<float4 *>(phic + 4 * j4) = make_float4(phi[0], phi[1], phi[2], phi[3]);
                if (SO && c == nchunks - 1)
                    *reinterpret_cast<float4 *>(slot_out + SLOT_PHIL + 4 * j4) =
                        make_float4(phi[0], phi[1], phi[2], phi[3]);
            }
            if (pt == 0) {
                mbar_arrive(bar(B_OPSREADY + ob));
                mbar_arrive(bar(B_BEMPTY + sb));
                mbar_arrive(bar(B_CEMPTY + scf));
            }
        }
        // the angle after the sequence's last token: phic after the last chunk
        // (every prep thread leaves the loop at the same chunk)
        if (last_seg && a.angle_out) {
            named_bar(1, PREP_THREADS);
            for (int k = pt; k < a.K; k += PREP_THREADS) a.angle_out[lane_id * a.K + k] = phic[k];
        }
    } else if (warp == W_XB) {
        // ------------------------------------------------------ X operands
        for (int c = 0; c < nchunks; c++) {
            const int sx = c % L::NXR, kx = c / L::NXR, scf = c % NC, kc = c / NC, ob = c & 1;
            if (!(warp_wait(bar(B_XFULL + sx), kx & 1, abort_flag, a.err, 8) &&
                  warp_wait(bar(B_CFULL + scf), kc & 1, abort_flag, a.err, 9) &&
                  (c < 2 || warp_wait(bar(B_OPSFREE + ob), ((c >> 1) - 1) & 1, abort_flag, a.err, 15))))
                break;
            const float *cf = coef0 + scf * CF_FLOATS;
            // the X operands, 16-byte vectors of 128-byte rows (a vector keeps its
            // place under the swizzle, so its row is its index / 8):
            //   SISO:  Xw = diag(xs) x
            //   MIMO:  Xr[(s,r)] = W_x[r] x_s (intra UMMA), Xw[(s,r)] = xs_s Xr[(s,r)]
            {
                const uint8_t *xt = sm + L::OFF_X + sx * L::SZ_X;
                uint4 *dw = reinterpret_cast<uint4 *>(sm + L::OFF_XW + ob * (Q * P * 2));
                uint4 *dr = reinterpret_cast<uint4 *>(sm + L::OFF_XR + ob * (Q * P * 2));
                // unrolled twice, not four times: measured 4 % faster calls
                // (the hot code of all roles shares the instruction cache)
#pragma unroll 2
                for (int v = l32; v < Q * P / 8; v += 32) {
                    const int row = v >> 3, pc = v & 7;
                    const int sq = row / R;                       // token of the row
                    const float sc = cf[CF_XS + sq];
                    uint4 d, dxr;
                    if (R == 1) {
                        d = reinterpret_cast<const uint4 *>(xt)[v];
                        uint32_t *w = reinterpret_cast<uint32_t *>(&d);
#pragma unroll
                        for (int q = 0; q < 4; q++) {
                            const float2 f = unpack_bf16(w[q]);
                            w[q] = pack_bf16(f.x * sc, f.y * sc);
                        }
                    } else {
                        const int rr = row % R;
                        const int cc = pc ^ (row & 7);            // logical 8-column chunk of this vector
                        const uint4 xv =
                            *reinterpret_cast<const uint4 *>(xt + sq * 128 + ((cc ^ (sq & 7)) << 4));
                        const uint32_t xw4[4] = {xv.x, xv.y, xv.z, xv.w};
                        uint32_t ow[4], orr[4];
#pragma unroll
                        for (int q = 0; q < 4; q++) {
                            const float2 f = unpack_bf16(xw4[q]);
                            const float x0 = f.x * wxs[rr * P + 8 * cc + 2 * q];
                            const float x1 = f.y * wxs[rr * P + 8 * cc + 2 * q + 1];
                            orr[q] = pack_bf16(x0, x1);
                            ow[q] = pack_bf16(x0 * sc, x1 * sc);
                        }
                        d = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                        dxr = make_uint4(orr[0], orr[1], orr[2], orr[3]);
                        if (!SO) dr[v] = dxr;
                    }
                    dw[v] = d;
                }
            }
            fence_async_smem();
            __syncwarp();
            if (l32 == 0) {
                mbar_arrive(bar(B_OPSREADY + ob));
                mbar_arrive(bar(B_XEMPTY + sx));
                mbar_arrive(bar(B_CEMPTY + scf));
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issue
        // The whole warp walks the chunks converged, so the descriptors are
        // warp-uniform; one elected lane issues each UMMA and commit.
        {
            const uint32_t id_kk = idesc(64, 64, 0, 0);    // D1 = Cbar . Bbar^T
            const uint32_t id_kmn = idesc(64, 64, 0, 1);   // D2, D3: B operand MN-major
            const uint32_t id_st = idesc(128, 64, 1, 1);   // D4: A and B MN-major
            // Descriptors are built once; a K-step of a UMMA only moves the start
            // address field (16-byte units, low bits of the descriptor).
            // (a buffer switch adds its byte offset / 16 to the start field)
            const uint64_t d_sp = sdesc(sbase + L::OFF_SP, 16, 1024);
            const uint64_t d_bb_k0 = sdesc(sbase + L::OFF_BB, 16, 1024);
            const uint64_t d_cb_k0 = sdesc(sbase + L::OFF_CB, 16, 1024);
            const uint64_t d_bb_mn0 = sdesc(sbase + L::OFF_BB, Q * 128, 1024);
            const uint64_t d_xw0 = sdesc(sbase + L::OFF_XW, Q * 128, 1024);
            const uint64_t d_xr0 = sdesc(sbase + L::OFF_XR, Q * 128, 1024);
            const uint64_t d_gb0 = sdesc(sbase + L::OFF_GB, N * 128, 1024);
            const uint64_t d_x0 = sdesc(sbase + L::OFF_X, Q * 128, 1024);
            constexpr uint64_t STEP_BC = (Q * N * 2) >> 4, STEP_XP = (Q * P * 2) >> 4, STEP_GB = SZ_GB >> 4;
            constexpr uint64_t STEP_X = L::SZ_X >> 4;
            // K-major operand, K-step kk of 16: 32 bytes inside a 128-byte atom row,
            // the second atom (K 64..127) Q*128 bytes further
            auto kstep_k = [](int kk) { return (uint64_t)(((kk >> 2) * (Q * 128) + (kk & 3) * 32) >> 4); };
            // MN-major operand, K-step kk of 16: two 8-row groups of 1024 bytes
            auto kstep_mn = [](int kk) { return (uint64_t)((kk * 2048) >> 4); };
            for (int c = 0; c < nchunks; c++) {
                const int sx = c % L::NXR, ob = c & 1;
                const uint64_t d_bb_k = d_bb_k0 + ob * STEP_BC, d_cb_k = d_cb_k0 + ob * STEP_BC;
                const uint64_t d_bb_mn = d_bb_mn0 + ob * STEP_BC, d_xw = d_xw0 + ob * STEP_XP;
                const uint64_t dx = (R == 1) ? d_x0 + (uint64_t)sx * STEP_X : d_xr0 + ob * STEP_XP;
                const uint64_t dg = d_gb0 + ((c + 1) & 1) * STEP_GB;   // state after chunk c-1
                if (!warp_wait_spin(bar(B_OPSREADY + ob), (c >> 1) & 1, abort_flag, a.err, 10)) break;
                if (SO) {
                    // state-only pass: the chunk-state UMMA alone
                    if (!warp_wait_spin(bar(B_STTAKEN), c & 1, abort_flag, a.err, 12)) break;
                    tc_fence_after();
                    if (elect_one()) {
                        for (int kk = 0; kk < Q / 16; kk++)
                            umma(tmem + COL_D4, d_bb_mn + kstep_mn(kk), d_xw + kstep_mn(kk), id_st, kk > 0);
                        umma_commit(bar(B_STFULL));
                        umma_commit(bar(B_OPSFREE + ob));
                    }
                    __syncwarp();
                    continue;
                }
                if (c > 0 && !warp_wait_spin(bar(B_STAKEN), (c - 1) & 1, abort_flag, a.err, 11)) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll 1
                    for (int kk = 0; kk < N / 16; kk++)
                        umma(tmem + COL_D1, d_cb_k + kstep_k(kk), d_bb_k + kstep_k(kk), id_kk, kk > 0);
                    umma_commit(bar(B_SFULL));
                }
                __syncwarp();
                if (!warp_wait_spin(bar(B_STTAKEN), c & 1, abort_flag, a.err, 12)) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll 1
                    for (int kk = 0; kk < Q / 16; kk++)
                        umma(tmem + COL_D4, d_bb_mn + kstep_mn(kk), d_xw + kstep_mn(kk), id_st, kk > 0);
                    umma_commit(bar(B_STFULL));
                }
                __syncwarp();
                // D3 buffer c & 1 was last read by the outputs of chunk c - 2
                if (c > 1 && !warp_wait_spin(bar(B_YTAKEN + (c & 1)), ((c >> 1) - 1) & 1, abort_flag, a.err, 13))
                    break;
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t d3 = tmem + COL_D3 + (uint32_t)(c & 1) * D3_STRIDE;
#pragma unroll 1
                    for (int kk = 0; kk < N / 16; kk++)
                        umma(d3, d_cb_k + kstep_k(kk), dg + kstep_mn(kk), id_kmn, kk > 0);
                    // SISO: B, C and Xw of chunk c are read by now (the intra UMMA
                    // reads the x tile and the scores only)
                    if (R == 1) umma_commit(bar(B_OPSFREE + ob));
                }
                __syncwarp();
                if (!warp_wait_spin(bar(B_SPFULL), c & 1, abort_flag, a.err, 14)) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll 1
                    for (int kk = 0; kk < Q / 16; kk++)
                        umma(tmem + COL_D2, d_sp + (uint64_t)((kk * 32) >> 4), dx + kstep_mn(kk), id_kmn, kk > 0);
                    umma_commit(bar(B_YFULL));
                    if (R > 1) umma_commit(bar(B_OPSFREE + ob));   // X_r is read by the intra UMMA
                    umma_commit(bar(B_XEMPTY + sx));
                }
                __syncwarp();
            }
            // drain: every MMA issued so far has completed before TMEM is freed
            if (elect_one()) umma_commit(bar(B_DRAIN));
            __syncwarp();
            const long long t0 = clock64();
            while (!mbar_try(bar(B_DRAIN), 0) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------- epilogue
        // Per chunk: mask the scores, fold the chunk state into g (this runs
        // while the intra UMMA completes), then write the outputs.
        const int q = warp & 3;                      // TMEM lane quarter
        const int ch = (warp - W_EPI0) >> 2;         // column half: 32 * ch .. 32 * ch + 31
        const int cb0 = 32 * ch;
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const int n = 32 * q + l32;                  // state row owned by this thread
        // score / output rows (M=64 accumulators, 16 lanes per quarter): this
        // thread holds rows ra and rb = ra + 8, two adjacent columns per group
        // of 8 (the 16x256b load layout)
        const int ra = 16 * q + (l32 >> 2), rb = ra + 8;
        const int ta = ra / R, tb = rb / R;          // their tokens
        const int cq = 2 * (l32 & 3);                // column offset inside a group of 8
        const int et = tid - W_EPI0 * 32;            // 0..255
        // my rows 16q..16q+15 against my columns 32ch..32ch+31 (tokens row / R,
        // col / R): wholly above the diagonal for ch = 1, q < 2; wholly below
        // it for ch = 0, q >= 2; across it otherwise (R = 1, 2, 4 alike)
        const bool blk_zero = ch == 1 && q < 2, blk_below = ch == 0 && q >= 2;
        const float Dh = a.D[h];
        uint8_t *sp = sm + L::OFF_SP;
        __nv_bfloat16 *yg = static_cast<__nv_bfloat16 *>(a.y);
        // each warp waits on its own (no group barrier): a warp that gives up
        // leaves its loop, and the others give up at their next wait
        auto group_wait = [&](int bi, uint32_t parity, int site) -> bool {
            return warp_wait(bar(bi), parity, abort_flag, a.err, site);
        };
        auto store_g = [&](const float *gv, int slot) {
            uint8_t *gb = sm + L::OFF_GB + slot * SZ_GB;
#pragma unroll
            for (int k4 = 0; k4 < 4; k4++) {
                const int cc = 4 * ch + k4;
                uint4 v;
                v.x = pack_bf16(gv[8 * k4], gv[8 * k4 + 1]);
                v.y = pack_bf16(gv[8 * k4 + 2], gv[8 * k4 + 3]);
                v.z = pack_bf16(gv[8 * k4 + 4], gv[8 * k4 + 5]);
                v.w = pack_bf16(gv[8 * k4 + 6], gv[8 * k4 + 7]);
                *reinterpret_cast<uint4 *>(gb + n * 128 + ((cc ^ (n & 7)) << 4)) = v;
            }
        };
        auto fold_state = [&](const float *cf, float *gv) {
            const float E = cf[CF_SCAL + 0];
#pragma unroll
            for (int c16 = 0; c16 < 2; c16++) {
                float d4[16];
                tmem_ld16(tl + COL_D4 + cb0 + 16 * c16, d4);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; u++) gv[16 * c16 + u] = fmaf(E, gv[16 * c16 + u], d4[u]);
            }
        };
        float g[32];
        if (SO) {
            // state-only pass: g starts at zero, only the state update runs
#pragma unroll
            for (int p = 0; p < 32; p++) g[p] = 0.f;
            __syncwarp();
            if (l32 == 0) mbar_arrive(bar(B_STTAKEN));
            float eacc = 1.f;
            bool ok2 = true;
            for (int c = 0; c < nchunks && ok2; c++) {
                const int scf = c % NC;
                const float *cf = coef0 + scf * CF_FLOATS;
                if (!(ok2 = group_wait(B_CFULL + scf, (c / NC) & 1, 24))) break;
                if (!(ok2 = group_wait(B_STFULL, c & 1, 25))) break;
                tc_fence_after();
                eacc *= cf[CF_SCAL + 0];
                fold_state(cf, g);
                tc_fence_before();
                __syncwarp();
                if (l32 == 0) {
                    mbar_arrive(bar(B_STTAKEN));
                    mbar_arrive(bar(B_CEMPTY + scf));
                }
            }
            if (!*abort_flag) {
                float *go = slot_out + SLOT_G + n * P + cb0;
#pragma unroll
                for (int p = 0; p < 32; p += 4)
                    *reinterpret_cast<float4 *>(go + p) = make_float4(g[p], g[p + 1], g[p + 2], g[p + 3]);
                if (et == 0) slot_out[SLOT_E] = eacc;
            }
        } else {
            {
                const int64_t base = (lane_id * N + n) * P + cb0;
                if (slot_in) {
                    // a later segment starts from the state the combine pass left in the slot
#pragma unroll
                    for (int p = 0; p < 32; p += 4) {
                        const float4 gv = *reinterpret_cast<const float4 *>(slot_in + SLOT_G + n * P + cb0 + p);
                        g[p] = gv.x; g[p + 1] = gv.y; g[p + 2] = gv.z; g[p + 3] = gv.w;
                    }
                } else {
                    const int64_t i0 = (b * Tn) * H + h;
                    const float f0 = (1.f - a.lam[i0]) * a.dt[i0];
#pragma unroll
                    for (int p = 0; p < 32; p += 4) {
                        const float4 hv = a.h0 ? *reinterpret_cast<const float4 *>(a.h0 + base + p)
                                               : make_float4(0, 0, 0, 0);
                        const float4 uv = a.prevBx0 ? *reinterpret_cast<const float4 *>(a.prevBx0 + base + p)
                                                    : make_float4(0, 0, 0, 0);
                        g[p] = fmaf(f0, uv.x, hv.x);
                        g[p + 1] = fmaf(f0, uv.y, hv.y);
                        g[p + 2] = fmaf(f0, uv.z, hv.z);
                        g[p + 3] = fmaf(f0, uv.w, hv.w);
                    }
                }
                store_g(g, 1);                       // read by the inter-chunk UMMA of chunk 0
                fence_async_smem();
                __syncwarp();
                if (l32 == 0) mbar_arrive(bar(B_STTAKEN));
            }
            bool ok = true;
            for (int c = 0; c < nchunks && ok; c++) {
                const int scf = c % NC, kc = c / NC, sx = c % L::NXR;
                const float *cf = coef0 + scf * CF_FLOATS;
                const uint8_t *xr = sm + L::OFF_X + sx * L::SZ_X;
                if (!(ok = group_wait(B_CFULL + scf, kc & 1, 20))) break;
                const bool unsafe = cf[CF_SCAL + 1] != 0.f;
                // ---- masked scores S' (rows ra, rb of D1; my 32 columns) ----
                // My 16 x 32 block of the 64 x 64 tile lies wholly above the
                // diagonal (zero: written at the first chunk, never again),
                // wholly below it (every score takes r_t e_s w_s), or across it.
                if (blk_zero) {
                    if (c == 0) {
#pragma unroll
                        for (int hf = 0; hf < 2; hf++)
#pragma unroll
                            for (int i = 0; i < 2; i++) {
                                const int col = cb0 + 16 * hf + 8 * i + cq, cc = col >> 3;
                                *reinterpret_cast<uint32_t *>(sp + ra * 128 + ((cc ^ (ra & 7)) << 4) + 2 * cq) = 0u;
                                *reinterpret_cast<uint32_t *>(sp + rb * 128 + ((cc ^ (rb & 7)) << 4) + 2 * cq) = 0u;
                            }
                    }
                } else {
                    if (!(ok = group_wait(B_SFULL, c & 1, 21))) break;
                    tc_fence_after();
                    const float rta = cf[CF_R + ta], gta = cf[CF_GAM + ta];
                    const float rtb = cf[CF_R + tb], gtb = cf[CF_GAM + tb];
#pragma unroll 1
                    for (int hf = 0; hf < 2; hf++) {
                        const int c0 = cb0 + 16 * hf;
                        float v[8];
                        tmem_ld16x256b_x2(tl + COL_D1 + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 2; i++) {
                            const int col = c0 + 8 * i + cq;
                            const int s0 = col / R, s1 = (col + 1) / R;   // tokens of the two columns
                            const float w0 = cf[CF_WM + s0], w1 = cf[CF_WM + s1];
                            if (blk_below) {
                                v[4 * i + 0] *= rta * w0;
                                v[4 * i + 1] *= rta * w1;
                                v[4 * i + 2] *= rtb * w0;
                                v[4 * i + 3] *= rtb * w1;
                            } else {
                                v[4 * i + 0] *= s0 < ta ? rta * w0 : (s0 == ta ? gta : 0.f);
                                v[4 * i + 1] *= s1 < ta ? rta * w1 : (s1 == ta ? gta : 0.f);
                                v[4 * i + 2] *= s0 < tb ? rtb * w0 : (s0 == tb ? gtb : 0.f);
                                v[4 * i + 3] *= s1 < tb ? rtb * w1 : (s1 == tb ? gtb : 0.f);
                                if (R == 1) {
                                    // SISO: the skip D x_t rides on the intra UMMA as D on the
                                    // diagonal of the scores (its B operand is x itself)
                                    v[4 * i + 0] += s0 == ta ? Dh : 0.f;
                                    v[4 * i + 1] += s1 == ta ? Dh : 0.f;
                                    v[4 * i + 2] += s0 == tb ? Dh : 0.f;
                                    v[4 * i + 3] += s1 == tb ? Dh : 0.f;
                                }
                            }
                            const int cc = col >> 3;
                            *reinterpret_cast<uint32_t *>(sp + ra * 128 + ((cc ^ (ra & 7)) << 4) + 2 * cq) =
                                pack_bf16(v[4 * i], v[4 * i + 1]);
                            *reinterpret_cast<uint32_t *>(sp + rb * 128 + ((cc ^ (rb & 7)) << 4) + 2 * cq) =
                                pack_bf16(v[4 * i + 2], v[4 * i + 3]);
                        }
                    }
                    if (unsafe) {
                        // exact path: the scores below the diagonal were stored
                        // unscaled; give each its factor e^{cum_t - cum_s} w_s here
#pragma unroll 1
                        for (int k = 0; k < 16; k++) {
                            const int row = (k & 2) ? rb : ra, t = row / R;
                            const int col = cb0 + 8 * (k >> 2) + cq + (k & 1), s2 = col / R;
                            if (s2 < t) {
                                __nv_bfloat16 *pv = reinterpret_cast<__nv_bfloat16 *>(sp + sw128(row, col));
                                const float m = exp2f(cf[CF_C2 + t] - cf[CF_C2 + s2]) * cf[CF_W + s2];
                                *pv = __float2bfloat16_rn(__bfloat162float(*pv) * m);
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
                // ---- state after chunk c: g = e^{cum_end} g + D4 (my 32 columns) ----
                if (!(ok = group_wait(B_STFULL, c & 1, 23))) break;
                tc_fence_after();
                fold_state(cf, g);
                tc_fence_before();
                store_g(g, c & 1);
                fence_async_smem();
                __syncwarp();
                if (l32 == 0) mbar_arrive(bar(B_STTAKEN));
                // ---- outputs y_t = sum_r W_y[r] (D2 + e^{cum_t} D3)_{(t,r)} + D x_t ----
                if (!(ok = group_wait(B_YFULL, c & 1, 22))) break;
                tc_fence_after();
                {
                    const float eca = cf[CF_EC + ta], ecb = cf[CF_EC + tb];
                    const int64_t tc0 = t_beg + (int64_t)c * QT;
#pragma unroll 1
                    for (int hf = 0; hf < 2; hf++) {
                        const int c0 = cb0 + 16 * hf;        // 16 columns: two groups of 8
                        float y2[8], y3[8];
                        tmem_ld16x256b_x2(tl + COL_D2 + c0, y2);
                        tmem_ld16x256b_x2(tl + COL_D3 + (uint32_t)(c & 1) * D3_STRIDE + c0, y3);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 2; i++) {
#pragma unroll
                            for (int j = 0; j < 4; j++) {
                                float v = fmaf((j & 2) ? ecb : eca, y3[4 * i + j], y2[4 * i + j]);
                                if (R > 1) {
                                    // contract the R rows of a token (threads l32 ^ 4, ^ 8) with W_y
                                    const int row = (j & 2) ? rb : ra;
                                    v *= wys[(row % R) * P + c0 + 8 * i + cq + (j & 1)];
#pragma unroll
                                    for (int o = 4; o < 4 * R; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                                }
                                y2[4 * i + j] = v;
                            }
                        }
#pragma unroll
                        for (int hb = 0; hb < 2; hb++) {
                            const int row = hb ? rb : ra, t = row / R;
                            if (row % R == 0 && tc0 + t < t_end) {
                                __nv_bfloat16 *yrow = yg + ((b * Tn + tc0 + t) * H + h) * P;
#pragma unroll
                                for (int i = 0; i < 2; i++) {
                                    const int col = c0 + 8 * i + cq, cc = col >> 3;
                                    float y0 = y2[4 * i + 2 * hb], y1 = y2[4 * i + 2 * hb + 1];
                                    if (R > 1) {   // SISO has D x in the intra term already
                                        const float2 xf = unpack_bf16(*reinterpret_cast<const uint32_t *>(
                                            xr + t * 128 + ((cc ^ (t & 7)) << 4) + 2 * cq));
                                        y0 = fmaf(Dh, xf.x, y0);
                                        y1 = fmaf(Dh, xf.y, y1);
                                    }
                                    *reinterpret_cast<uint32_t *>(yrow + col) = pack_bf16(y0, y1);
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (l32 == 0) {
                    mbar_arrive(bar(B_YTAKEN + (c & 1)));
                    if (R > 1) mbar_arrive(bar(B_XEMPTY + sx));
                    mbar_arrive(bar(B_CEMPTY + scf));
                }
            }
            // final state: h_{T-1} = g after the last chunk (no lookahead there)
            if (!*abort_flag && a.h_out && last_seg) {
                float *ho = a.h_out + (lane_id * N + n) * P + cb0;
#pragma unroll
                for (int p = 0; p < 32; p += 4)
                    *reinterpret_cast<float4 *>(ho + p) = make_float4(g[p], g[p + 1], g[p + 2], g[p + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // prev_Bx = sum_r Bbar_{T-1,r} X_{T-1,r}^T (rotated, unscaled B rows kept by
    // the rotation warps; X_{T-1,r} = W_x[r] x_{T-1})
    if (!SO && last_seg && !*abort_flag && a.prevBx_out && warp >= W_EPI0 && warp < W_EPI0 + EPI_WARPS) {
        const int et = tid - W_EPI0 * 32;
        const int n = et & (N - 1), half = et >> 7;
        const int c = nchunks - 1;
        const int Lc = (int)(t_end - t_beg - (int64_t)c * QT);
        const uint8_t *xr = sm + L::OFF_X + (c % L::NXR) * L::SZ_X;
        const int t = Lc - 1;
        float *uo = a.prevBx_out + (lane_id * N + n) * P;
        for (int cc = 4 * half; cc < 4 * half + 4; cc++) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(xr + t * 128 + ((cc ^ (t & 7)) << 4));
            const uint32_t xw4[4] = {xv.x, xv.y, xv.z, xv.w};
            float o[8];
            for (int e2 = 0; e2 < 4; e2++) {
                const float2 f = unpack_bf16(xw4[e2]);
                const int p = 8 * cc + 2 * e2;
                float u0 = 0.f, u1 = 0.f;
                for (int r = 0; r < R; r++) {
                    const float bn = blast[r * N + n];
                    const float w0 = (R > 1) ? wxs[r * P + p] : 1.f, w1 = (R > 1) ? wxs[r * P + p + 1] : 1.f;
                    u0 += bn * w0 * f.x;
                    u1 += bn * w1 * f.y;
                }
                o[2 * e2] = u0;
                o[2 * e2 + 1] = u1;
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

// 4-D map over a (Bt, T, H, inner) tensor: dims (inner, H, T, Bt); with
// rank > 0 a 5-D map over (Bt, T, H, rank, inner): dims (inner, rank, H, T, Bt)
// whose box holds every rank.
static bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int64_t inner,
                     int64_t H, int64_t T, int64_t Bt, uint32_t box_inner, uint32_t box_t, CUtensorMapSwizzle sw,
                     int64_t rank = 0) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (rank > 0) {
        cuuint64_t dims[5] = {(cuuint64_t)inner, (cuuint64_t)rank, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)Bt};
        cuuint64_t strides[4] = {(cuuint64_t)(inner * esize), (cuuint64_t)(inner * rank * esize),
                                 (cuuint64_t)(inner * rank * H * esize), (cuuint64_t)(inner * rank * H * T * esize)};
        cuuint32_t box[5] = {box_inner, (cuuint32_t)rank, 1, box_t, 1};
        return fn(m, dt, 5, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)Bt};
    cuuint64_t strides[3] = {(cuuint64_t)(inner * esize), (cuuint64_t)(inner * H * esize),
                             (cuuint64_t)(inner * H * T * esize)};
    cuuint32_t box[4] = {box_inner, 1, box_t, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__device__ int g_tc_error;

// Segment plan: when there are too few (b, h) lanes to fill the GPU, each
// lane's sequence is cut into segments of whole chunks that run in parallel.
struct SegPlan {
    int nseg;
    int64_t seg_len;
};
static SegPlan seg_plan(int64_t lanes, int64_t T) {
    SegPlan p{1, T};
    if (lanes >= 96 || T <= 8 * Q) return p;
    // A CTA holds a whole SM (shared memory), so a pass over k CTAs takes
    // ceil(k / 148) waves of (chunks per segment) chunk times; the state-only
    // pass over the nseg - 1 leading segments costs about 0.6 of a full chunk
    // per chunk.  Pick the segment count with the least time in those units,
    // with at least 4 chunks per segment and the workspace ((nseg - 1) * lanes
    // slots) within 24 MB.
    const int64_t nq = (T + Q - 1) / Q;
    const int64_t max_slots = ((int64_t)24 << 20) / ((int64_t)SLOT_FLOATS * 4);
    auto waves = [](int64_t ctas) { return (ctas + 147) / 148; };
    double best = (double)waves(lanes) * (double)nq;
    for (int64_t ns = 2; ns <= 64; ns++) {
        const int64_t len_q = (nq + ns - 1) / ns;
        if (len_q < 4) break;
        const int64_t nsr = (nq + len_q - 1) / len_q;   // segments at that length
        if (nsr < 2 || (nsr - 1) * lanes > max_slots) continue;
        const double cost = ((double)waves(lanes * nsr) + 0.6 * (double)waves(lanes * (nsr - 1))) * (double)len_q;
        if (cost < best - 1e-9) {
            best = cost;
            p.nseg = (int)nsr;
            p.seg_len = len_q * Q;
        }
    }
    return p;
}

// Chains the segments of every lane: the state entering segment j+1 is
//   g_in(j+1) = A_j g_in(j) + R(Phi_in(j)) g_loc(j),   Phi_in(j+1) = Phi_in(j) + dPhi_j
// where g_loc(j) is segment j's end state from a zero start in its own angle
// frame, A_j its decay product and R rotates every pair of state rows (2i,
// 2i+1) by the angle of pair i (the rotation moves the local frame to the
// absolute one: Bbar = R(Phi_in + phi_local) B).  One thread per (pair, column).
__global__ void __launch_bounds__(256) k_seg_combine(TcArgs a) {
    const int64_t lane = blockIdx.x, b = lane / a.H, h = lane % a.H;
    const int idx = blockIdx.y * 256 + threadIdx.x;
    const int i = idx / P, p = idx % P;
    const int64_t i0 = (b * a.T) * a.H + h;
    const float f0 = (1.f - a.lam[i0]) * a.dt[i0];
    const int64_t r0 = (lane * N + 2 * i) * P + p, r1 = r0 + P;
    float g0 = (a.h0 ? a.h0[r0] : 0.f) + f0 * (a.prevBx0 ? a.prevBx0[r0] : 0.f);
    float g1 = (a.h0 ? a.h0[r1] : 0.f) + f0 * (a.prevBx0 ? a.prevBx0[r1] : 0.f);
    float phi = (a.angle0 && i < a.K) ? a.angle0[lane * a.K + i] : 0.f;
    for (int j = 0; j < a.nseg - 1; j++) {
        float *sl = a.ws + ((size_t)lane * (a.nseg - 1) + j) * SLOT_FLOATS;
        const float l0 = sl[SLOT_G + 2 * i * P + p], l1 = sl[SLOT_G + (2 * i + 1) * P + p];
        const float E = sl[SLOT_E], dphi = sl[SLOT_PHIL + i];
        float sn, cs;
        sincosf(phi, &sn, &cs);
        g0 = fmaf(E, g0, cs * l0 - sn * l1);
        g1 = fmaf(E, g1, sn * l0 + cs * l1);
        sl[SLOT_G + 2 * i * P + p] = g0;
        sl[SLOT_G + (2 * i + 1) * P + p] = g1;
        phi += dphi;
        if (p == 0) sl[SLOT_PHIN + i] = phi;
    }
}

// Exercises the timeout path of the bounded waits without any fault: one
// thread waits, with the kernels' own bounded wait, on an mbarrier that
// nothing ever arrives on.  The wait gives up after WAIT_LIMIT_CYCLES, sets
// the abort flag, records `site` in the device error word and the kernel
// returns normally.
__global__ void k_wait_selftest(int *err, int site) {
    __shared__ alignas(8) uint64_t never;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&never), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)wait_bar(smem_u32(&never), 0, &abort_flag, err, site);
    __syncthreads();
}

}  // namespace tc

cudaError_t launch_wait_selftest(int site, cudaStream_t s) {
    int *err = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&err), tc::g_tc_error);
    if (e != cudaSuccess) return e;
    tc::k_wait_selftest<<<1, 32, 0, s>>>(err, site);
    count_launch();
    return cudaGetLastError();
}

size_t scan_tc_workspace_bytes(int64_t Bt, int64_t H, int64_t T) {
    const tc::SegPlan pl = tc::seg_plan(Bt * H, T);
    if (pl.nseg <= 1) return 0;
    return (size_t)(Bt * H) * (size_t)(pl.nseg - 1) * tc::SLOT_FLOATS * sizeof(float);
}

// The kernel's chunk is 64 rows: 64 tokens (SISO) or 64 / R tokens of R
// ranks (MIMO, R = 2 or 4).  A requested chunk that is a multiple of that runs
// as sub-chunks (the same result up to rounding order).
bool scan_tc_supported(const ScanArgs &a, m3_dtype dt) {
    const bool shape = a.mimo_layout ? (a.R == 2 || a.R == 4) : (a.R == 1);
    return dt == M3_BF16 && shape && a.P == tc::P && a.N == tc::N && a.Q > 0 && a.Q % (tc::Q / a.R) == 0 &&
           a.K % 4 == 0 && a.K > 0 && a.G > 0 &&
           a.T > 0 && a.T <= ((int64_t)1 << 30) && a.Bt <= 65535 && a.H <= 65535;
}

template <int R>
static cudaError_t launch_tc_r(const ScanArgs &a, cudaStream_t s) {
    using namespace tc;
    constexpr int QT = Q / R;
    CUtensorMap mx, mb, mc, mth;
    const int64_t rk = R > 1 ? R : 0;
    if (!make_map(&mx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P, a.H, a.T, a.Bt, P, QT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mb, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, a.G, a.T, a.Bt, N, QT, CU_TENSOR_MAP_SWIZZLE_NONE,
                  rk) ||
        !make_map(&mc, a.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, a.G, a.T, a.Bt, N, QT, CU_TENSOR_MAP_SWIZZLE_NONE,
                  rk) ||
        !make_map(&mth, a.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.K, a.H, a.T, a.Bt, (uint32_t)a.K, QT,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    TcArgs t;
    t.y = a.y;
    t.theta = a.theta;
    t.dt = a.dt; t.A = a.A; t.lam = a.lam; t.D = a.D;
    t.Wx = a.Wx; t.Wy = a.Wy;
    t.h0 = a.h0; t.prevBx0 = a.prevBx0; t.angle0 = a.angle0;
    t.nrm = a.nrm;
    t.h_out = a.h_out; t.prevBx_out = a.prevBx_out; t.angle_out = a.angle_out;
    t.Bt = a.Bt; t.T = a.T; t.H = a.H; t.G = a.G; t.K = (int)a.K;
    const SegPlan pl = seg_plan(a.Bt * a.H, a.T);
    t.nseg = pl.nseg;
    t.seg_len = pl.seg_len;
    t.ws = static_cast<float *>(a.ws);
    int *err = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&err), g_tc_error);
    if (e != cudaSuccess) return e;
    t.err = err;
    const int64_t lanes = a.Bt * a.H;
    constexpr int SMEM = smem_bytes<R>();
    if (pl.nseg > 1) {
        cudaFuncSetAttribute(k_scan_tc<true, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        k_scan_tc<true, R><<<(unsigned)(lanes * (pl.nseg - 1)), THREADS, SMEM, s>>>(mx, mb, mc, mth, t);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_seg_combine<<<dim3((unsigned)lanes, NP2 * P / 256), 256, 0, s>>>(t);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cudaFuncSetAttribute(k_scan_tc<false, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    k_scan_tc<false, R><<<(unsigned)(lanes * pl.nseg), THREADS, SMEM, s>>>(mx, mb, mc, mth, t);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t s) {
    switch (a.R) {
        case 1: return launch_tc_r<1>(a, s);
        case 2: return launch_tc_r<2>(a, s);
        case 4: return launch_tc_r<4>(a, s);
    }
    return cudaErrorInvalidValue;
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
