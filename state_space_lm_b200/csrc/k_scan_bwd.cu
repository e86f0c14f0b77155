// k_scan_bwd.cu -- backward of the chunked Mamba-3 scan (SISO and rank-R
// MIMO, grouped B/C, partial RoPE, QkNorm and BC-bias) on the fp32 FFMA pipes.
//
// Training needs the gradient of the scan (TorchMamba README, "Models" and
// "Verification").  The forward is the shifted-state form of the chunked
// kernels (dotLLM pull request, "Stage A: Mamba3SelectiveScan" and the
// streaming-decode comment): g_t = alpha_t g_{t-1} + w_t U_t with
// w_t = gamma_t + (1-lam_{t+1}) dt_{t+1}, g_{-1} = h0 + (1-lam_0) dt_0 prev_Bx0,
// h_t = alpha_t g_{t-1} + gamma_t U_t, y_t = sum_r W_y[r] (Cbar_{t,r}^T h_t)
// + D x_t, h_final = g_{T-1}, prev_Bx_final = U_{T-1}.  Inside a chunk with
// entering state g_in, running log-decay cum_t and Gin the adjoint of the
// chunk's last g (dh_final for the last chunk):
//   Dy_{s,r}  = W_y[r] dy_s,  X_{t,r} = W_x[r] x_t,  M[s,t] = e^{cum_s-cum_t} w_t
//               (t < s), gamma_s (t = s)
//   dX_{t,r}  = sum_{s>=t} M[s,t] sum_r' (Cbar_{s,r'}.Bbar_{t,r}) Dy_{s,r'}
//               + w_t e^{cum_end-cum_t} Bbar_{t,r}^T Gin
//   dBbar_{t,r} = sum_{s>=t} M[s,t] sum_r' (Dy_{s,r'}.X_{t,r}) Cbar_{s,r'}
//               + w_t e^{cum_end-cum_t} Gin X_{t,r}
//   dCbar_{s,r'} = sum_{t<=s} M[s,t] sum_r (Dy_{s,r'}.X_{t,r}) Bbar_{t,r}
//               + e^{cum_s} g_in Dy_{s,r'}
//   dM[s,t]   = sum_{r',r} (Cbar_{s,r'}.Bbar_{t,r}) (Dy_{s,r'}.X_{t,r})
//   Gin(prev chunk) = e^{cum_end} Gin + sum_{s,r} e^{cum_s} Cbar_{s,r} Dy_{s,r}^T
// and the mask, decay and lookahead adjoints follow from M, from the inter
// term e^{cum_s} Cbar_s^T g_in and from g_out = e^{cum_end} g_in +
// sum_t e^{cum_end-cum_t} w_t U_t.  The rotation by Phi_t turns the pair
// adjoints back by -Phi_t and feeds the angle adjoint, which runs backwards
// over the whole sequence (dtheta_t = dt_t GPhi_t); QkNorm and the bias
// are undone per row.
//
// Three launches:
//   k_bwd_state   one CTA per (b, h) lane walks the chunks forward and keeps
//                 each chunk's entering state g_in and angle in the workspace;
//   k_bwd_chunks  one CTA per lane walks the chunks backwards;
//   k_bwd_params  sums the per-lane partial gradients of the shared
//                 parameters (A, D, W_x, W_y, gains, biases) over the batch
//                 and, when B/C are grouped, the heads of each group.
// Every sum runs in a fixed order, so the result is deterministic.
#include "m3_internal.cuh"

namespace m3 {

// ---- shared-memory layout of one lane (floats) ----------------------------
// Rows of B, C, their adjoints (N padded to a multiple of 4, stride Np + 4)
// and of X, Dy (stride Pp + 4); the states are kept transposed, (P, Np + 4),
// so that every small product below reads conflict-free 16-byte vectors.
struct BwdLayout {
    int Q, QR, Np, Pp, ldn, ldp, ldq;
    size_t Bb, Cb, dBb, dCb, X, Dy, BG, CG, S, V, DM, MK, gs, Gs, Ph, GP, tok, inv, rsc, par, misc, total;
};

enum {  // per-token scalar arrays, each Q floats
    TK_DT, TK_LAM, TK_LA, TK_CUM, TK_GAM, TK_W, TK_EC, TK_CS, TK_Q, TK_YI, TK_DCUM, TK_DW, TK_DLA, TK_DTH,
    TK_DYX, TK_DGAM, TK_CW, TK_COUNT
};

__host__ __device__ inline size_t par_floats(int64_t P, int64_t N, int64_t R) {
    return 2 + 2 * (size_t)R * P + 2 * (size_t)N + 2 * (size_t)R * N;
}

__host__ __device__ inline BwdLayout bwd_layout(int64_t P, int64_t N, int64_t R, int64_t K, int Q) {
    BwdLayout L;
    L.Q = Q;
    L.QR = Q * (int)R;
    L.Np = (int)((N + 3) & ~3);
    L.Pp = (int)((P + 3) & ~3);
    L.ldn = L.Np + 4;
    L.ldp = L.Pp + 4;
    L.ldq = ((L.QR + 3) & ~3) + 4;   // row stride of the (rows x rows) score matrices
    auto al4 = [](size_t v) { return (v + 3) & ~(size_t)3; };
    size_t o = 0;
    const size_t QRp = (size_t)((L.QR + 3) & ~3);   // rows rounded up: 4-row products read whole groups
    const size_t rowsN = QRp * L.ldn, rowsP = QRp * L.ldp, st = (size_t)L.Pp * L.ldn;
    L.Bb = o; o += rowsN;
    L.Cb = o; o += rowsN;
    L.dBb = o; o += rowsN;
    L.dCb = o; o += rowsN;
    L.X = o; o += rowsP;
    L.Dy = o; o += rowsP;
    L.BG = o; o += rowsP;
    L.CG = o; o += rowsP;
    L.gs = o; o += st;
    L.Gs = o; o += st;
    L.S = o; o += (size_t)L.QR * L.ldq;
    L.V = o; o += (size_t)L.QR * L.ldq;
    L.DM = o; o += al4((size_t)Q * Q);
    L.MK = o; o += al4((size_t)Q * Q);
    L.Ph = o; o += al4((size_t)Q * K);
    L.GP = o; o += al4((size_t)Q * K);
    L.tok = o; o += al4((size_t)TK_COUNT * Q);
    L.inv = o; o += al4(2 * (size_t)L.QR);
    L.rsc = o; o += al4(2 * (size_t)L.QR);
    L.par = o; o += al4(par_floats(P, N, R));
    L.misc = o; o += al4(2 * (size_t)K + 32 + 8);
    L.total = o;
    return L;
}

// Per-lane partial sums of the shared parameters: dA, dD, dW_x (R*P),
// dW_y (R*P), the B and C gains (N each), the B and C biases (R*N each).
struct ParOff {
    size_t Wx, Wy, wB, wC, bB, bC;
    __host__ __device__ ParOff(int64_t P, int64_t N, int64_t R) {
        Wx = 2;
        Wy = Wx + (size_t)R * P;
        wB = Wy + (size_t)R * P;
        wC = wB + (size_t)N;
        bB = wC + (size_t)N;
        bC = bB + (size_t)R * N;
    }
};

// Largest chunk <= the requested one (and <= 64) whose layout fits 220 KB.
int bwd_chunk(int64_t P, int64_t N, int64_t R, int64_t K, int64_t chunk) {
    constexpr size_t limit = 220 * 1024;
    int q = (int)(chunk < 64 ? chunk : 64);
    while (q > 1 && sizeof(float) * bwd_layout(P, N, R, K, q).total > limit) q = (q + 1) / 2;
    if (sizeof(float) * bwd_layout(P, N, R, K, q).total > limit) return 0;
    return q;
}

// Workspace: per (lane, chunk) the entering state g_in (N*P, row-major) and
// angle (K); per lane the partial sums; per head the B/C gradients when grouped.
struct BwdWs {
    size_t slots, partial, dBh, dCh, total;  // offsets in floats
};
static BwdWs bwd_ws(const BwdArgs &a, int Q) {
    BwdWs w;
    const int64_t lanes = a.Bt * a.H, nch = (a.T + Q - 1) / Q;
    size_t o = 0;
    w.slots = o; o += (size_t)lanes * nch * (a.N * a.P + a.K);
    w.partial = o; o += (size_t)lanes * par_floats(a.P, a.N, a.R);
    const size_t bc = (a.G < a.H) ? (size_t)a.Bt * a.T * a.H * a.R * a.N : 0;
    w.dBh = o; o += bc;
    w.dCh = o; o += bc;
    w.total = o;
    return w;
}

size_t scan_bwd_workspace_bytes(const BwdArgs &a) {
    const int q = bwd_chunk(a.P, a.N, a.R, a.K, a.Q);
    if (q < 1) return 0;
    return sizeof(float) * bwd_ws(a, q).total;
}

struct BwdSmem {
    float *Bb, *Cb, *dBb, *dCb, *X, *Dy, *BG, *CG, *S, *V, *DM, *MK, *gs, *Gs, *Ph, *GP, *tok, *inv, *rsc, *par, *misc;
    __device__ BwdSmem(float *sm, const BwdLayout &L)
        : Bb(sm + L.Bb), Cb(sm + L.Cb), dBb(sm + L.dBb), dCb(sm + L.dCb), X(sm + L.X), Dy(sm + L.Dy),
          BG(sm + L.BG), CG(sm + L.CG), S(sm + L.S), V(sm + L.V), DM(sm + L.DM), MK(sm + L.MK), gs(sm + L.gs),
          Gs(sm + L.Gs), Ph(sm + L.Ph), GP(sm + L.GP), tok(sm + L.tok), inv(sm + L.inv), rsc(sm + L.rsc),
          par(sm + L.par), misc(sm + L.misc) {}
    __device__ float *tk(int k, int Q) const { return tok + k * Q; }
};

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}
__device__ __forceinline__ float4 axpy4(float s, float4 x, float4 y) {
    return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}

// ---- the three small products (register tiles, conflict-free vectors) -----
// out[row][p] = sum_n A[row][n] St[p][n]   (rows < nrows, p < P; A, St padded with zeros to Np)
// A warp shares its 4 rows and owns 64 columns p (lanes, lanes + 32).
__device__ void mm_rows_by_state(const float *A, int lda, int nrows, const float *St, int lds, int Np, int P,
                                 float *out, int ldo) {
    const int nrb = (nrows + 3) / 4, npb = (P + 63) / 64;
    for (int it = threadIdx.x; it < nrb * npb * 32; it += blockDim.x) {
        const int l = it & 31, q = it >> 5, pb = q % npb, r0 = (q / npb) * 4;
        const int p0 = pb * 64 + l, p1 = p0 + 32;
        const float *s0 = St + (size_t)(p0 < P ? p0 : 0) * lds, *s1 = St + (size_t)(p1 < P ? p1 : 0) * lds;
        const float *a0 = A + (size_t)min(r0, nrows - 1) * lda, *a1 = A + (size_t)min(r0 + 1, nrows - 1) * lda;
        const float *a2 = A + (size_t)min(r0 + 2, nrows - 1) * lda, *a3 = A + (size_t)min(r0 + 3, nrows - 1) * lda;
        float c00 = 0.f, c01 = 0.f, c10 = 0.f, c11 = 0.f, c20 = 0.f, c21 = 0.f, c30 = 0.f, c31 = 0.f;
#pragma unroll 2
        for (int n = 0; n < Np; n += 4) {
            const float4 b0 = ld4(s0 + n), b1 = ld4(s1 + n);
            float4 v = ld4(a0 + n);
            c00 = dot4(v, b0, c00); c01 = dot4(v, b1, c01);
            v = ld4(a1 + n);
            c10 = dot4(v, b0, c10); c11 = dot4(v, b1, c11);
            v = ld4(a2 + n);
            c20 = dot4(v, b0, c20); c21 = dot4(v, b1, c21);
            v = ld4(a3 + n);
            c30 = dot4(v, b0, c30); c31 = dot4(v, b1, c31);
        }
        const float cc[4][2] = {{c00, c01}, {c10, c11}, {c20, c21}, {c30, c31}};
#pragma unroll
        for (int j = 0; j < 4; j++)
            if (r0 + j < nrows) {
                if (p0 < P) out[(size_t)(r0 + j) * ldo + p0] = cc[j][0];
                if (p1 < P) out[(size_t)(r0 + j) * ldo + p1] = cc[j][1];
            }
    }
}

// out[row][n..n+3] = sum_p X[row][p] St[p][n..n+3]   (rows < nrows, n < Np)
// A warp shares its 4 rows and owns 32 groups of 4 columns n.
__device__ void mm_rows_by_stateT(const float *X, int ldx, int nrows, const float *St, int lds, int Np, int P,
                                  float *out, int ldo) {
    const int ngt = Np / 4, nnb = (ngt + 31) / 32, nrb = (nrows + 3) / 4;
    for (int it = threadIdx.x; it < nrb * nnb * 32; it += blockDim.x) {
        const int l = it & 31, q = it >> 5, nb = q % nnb, r0 = (q / nnb) * 4;
        const int ng = nb * 32 + l;
        const float *sp = St + 4 * (ng < ngt ? ng : 0);
        const float *x0 = X + (size_t)min(r0, nrows - 1) * ldx, *x1 = X + (size_t)min(r0 + 1, nrows - 1) * ldx;
        const float *x2 = X + (size_t)min(r0 + 2, nrows - 1) * ldx, *x3 = X + (size_t)min(r0 + 3, nrows - 1) * ldx;
        float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f), c1 = c0, c2 = c0, c3 = c0;
#pragma unroll 4
        for (int p = 0; p < P; p++) {
            const float4 sv = ld4(sp + (size_t)p * lds);
            c0 = axpy4(x0[p], sv, c0);
            c1 = axpy4(x1[p], sv, c1);
            c2 = axpy4(x2[p], sv, c2);
            c3 = axpy4(x3[p], sv, c3);
        }
        if (ng < ngt) {
            if (r0 < nrows) st4(out + (size_t)r0 * ldo + 4 * ng, c0);
            if (r0 + 1 < nrows) st4(out + (size_t)(r0 + 1) * ldo + 4 * ng, c1);
            if (r0 + 2 < nrows) st4(out + (size_t)(r0 + 2) * ldo + 4 * ng, c2);
            if (r0 + 3 < nrows) st4(out + (size_t)(r0 + 3) * ldo + 4 * ng, c3);
        }
    }
}

// St[p][n] <- e St[p][n] + sum_{row < nrows} A[row][n] coef[row / R] Y[row][p]
// A warp owns 32 groups of 4 columns n and shares its 8 columns p.
__device__ void mm_state_update(float *St, int lds, int Np, int P, float e, const float *A, int lda,
                                const float *Y, int ldy, const float *coef, int R, int nrows) {
    constexpr int TP = 8;
    const int ngt = Np / 4, nnb = (ngt + 31) / 32, npb = (P + TP - 1) / TP;
    for (int it = threadIdx.x; it < nnb * npb * 32; it += blockDim.x) {
        const int l = it & 31, q = it >> 5, nb = q % nnb, p0 = (q / nnb) * TP;
        const int ng = nb * 32 + l, n4 = 4 * (ng < ngt ? ng : 0);
        float4 acc[TP];
#pragma unroll
        for (int k = 0; k < TP; k++)
            acc[k] = (p0 + k < P) ? make_float4(e * St[(size_t)(p0 + k) * lds + n4], e * St[(size_t)(p0 + k) * lds + n4 + 1],
                                                e * St[(size_t)(p0 + k) * lds + n4 + 2], e * St[(size_t)(p0 + k) * lds + n4 + 3])
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int row = 0; row < nrows; row++) {
            const float c = coef[row / R];
            const float4 av = ld4(A + (size_t)row * lda + n4);
            const float *yr = Y + (size_t)row * ldy + p0;
#pragma unroll
            for (int k = 0; k < TP; k++) acc[k] = axpy4(c * yr[k < P - p0 ? k : 0], av, acc[k]);
        }
        if (ng < ngt) {
#pragma unroll
            for (int k = 0; k < TP; k++)
                if (p0 + k < P) st4(St + (size_t)(p0 + k) * lds + n4, acc[k]);
        }
    }
}

// out[c][j..j+1] = rs[c/R] out[c][j..j+1] + sum_{k < nk} W[k][c] Rm[k][j..j+1]
// (W read by columns: a warp shares 4 output rows c, its lanes own column pairs j)
__device__ void mm_wT_rows(float *out, int ldo, int nrows, const float *W, int ldw, int nk, const float *Rm, int ldr,
                           int ncols, const float *rs, int R) {
    const int ngt = ncols / 2, njb = (ngt + 31) / 32, nrb = (nrows + 3) / 4;
    for (int it = threadIdx.x; it < nrb * njb * 32; it += blockDim.x) {
        const int l = it & 31, q = it >> 5, jb = q % njb, c0 = (q / njb) * 4;
        const int jg = jb * 32 + l, j = 2 * (jg < ngt ? jg : 0);
        float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
        for (int k = 0; k < nk; k++) {
            const float2 r = *reinterpret_cast<const float2 *>(Rm + (size_t)k * ldr + j);
            const float4 wv = ld4(W + (size_t)k * ldw + c0);
            a0.x = fmaf(wv.x, r.x, a0.x); a0.y = fmaf(wv.x, r.y, a0.y);
            a1.x = fmaf(wv.y, r.x, a1.x); a1.y = fmaf(wv.y, r.y, a1.y);
            a2.x = fmaf(wv.z, r.x, a2.x); a2.y = fmaf(wv.z, r.y, a2.y);
            a3.x = fmaf(wv.w, r.x, a3.x); a3.y = fmaf(wv.w, r.y, a3.y);
        }
        if (jg < ngt) {
            const float2 av[4] = {a0, a1, a2, a3};
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (c0 + i < nrows) {
                    float2 *o = reinterpret_cast<float2 *>(out + (size_t)(c0 + i) * ldo + j);
                    const float sc = rs[(c0 + i) / R];
                    *o = make_float2(fmaf(sc, o->x, av[i].x), fmaf(sc, o->y, av[i].y));
                }
        }
    }
}

// out[r][j..j+1] = rs[r/R] out[r][j..j+1] + sum_{k < nk} W[r][k] Rm[k][j..j+1]
// (nk rounded up to 4: W's columns from nk on must be zero; a warp shares 4 rows r)
__device__ void mm_w_rows(float *out, int ldo, int nrows, const float *W, int ldw, int nk, const float *Rm, int ldr,
                          int ncols, const float *rs, int R) {
    const int ngt = ncols / 2, njb = (ngt + 31) / 32, nrb = (nrows + 3) / 4, nk4 = (nk + 3) & ~3;
    for (int it = threadIdx.x; it < nrb * njb * 32; it += blockDim.x) {
        const int l = it & 31, q = it >> 5, jb = q % njb, r0 = (q / njb) * 4;
        const int jg = jb * 32 + l, j = 2 * (jg < ngt ? jg : 0);
        float2 acc[4];
#pragma unroll
        for (int i = 0; i < 4; i++) acc[i] = make_float2(0.f, 0.f);
        for (int k = 0; k < nk4; k += 4) {
            float2 rk[4];
#pragma unroll
            for (int u = 0; u < 4; u++) rk[u] = *reinterpret_cast<const float2 *>(Rm + (size_t)(k + u) * ldr + j);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float4 wv = ld4(W + (size_t)min(r0 + i, nrows - 1) * ldw + k);
                acc[i].x = fmaf(wv.x, rk[0].x, fmaf(wv.y, rk[1].x, fmaf(wv.z, rk[2].x, fmaf(wv.w, rk[3].x, acc[i].x))));
                acc[i].y = fmaf(wv.x, rk[0].y, fmaf(wv.y, rk[1].y, fmaf(wv.z, rk[2].y, fmaf(wv.w, rk[3].y, acc[i].y))));
            }
        }
        if (jg < ngt) {
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (r0 + i < nrows) {
                    float2 *o = reinterpret_cast<float2 *>(out + (size_t)(r0 + i) * ldo + j);
                    const float sc = rs[(r0 + i) / R];
                    *o = make_float2(fmaf(sc, o->x, acc[i].x), fmaf(sc, o->y, acc[i].y));
                }
        }
    }
}

// S[rr][cr] = Cbar_rr . Bbar_cr and V[rr][cr] = Dy_rr . X_cr for token(cr) <= token(rr), else 0
// (lanes own consecutive rows rr -- conflict-free 16-byte loads -- and a warp shares 4 columns cr)
__device__ void scores(float *S, float *V, int ldq, const float *Cb, const float *Bb, int ldn, int Np, const float *Dy,
                       const float *X, int ldp, int Pp, int nrows, int R) {
    const int nrb = (nrows + 31) / 32, ncg = (nrows + 3) / 4;
    for (int it = threadIdx.x; it < ncg * nrb * 32; it += blockDim.x) {
        const int l = it & 31, q = it >> 5, rb = q % nrb, c0 = (q / nrb) * 4;
        const int rr = rb * 32 + l;
        const int rc = min(rr, nrows - 1);
        if (c0 / R > rc / R) {   // the whole tile lies above the diagonal
            if (rr < nrows) {
                st4(S + (size_t)rr * ldq + c0, make_float4(0.f, 0.f, 0.f, 0.f));
                st4(V + (size_t)rr * ldq + c0, make_float4(0.f, 0.f, 0.f, 0.f));
            }
            continue;
        }
        const float *cp = Cb + (size_t)rc * ldn, *dp = Dy + (size_t)rc * ldp;
        const float *b0 = Bb + (size_t)min(c0, nrows - 1) * ldn, *b1 = Bb + (size_t)min(c0 + 1, nrows - 1) * ldn;
        const float *b2 = Bb + (size_t)min(c0 + 2, nrows - 1) * ldn, *b3 = Bb + (size_t)min(c0 + 3, nrows - 1) * ldn;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        for (int n = 0; n < Np; n += 4) {
            const float4 cv = ld4(cp + n);
            s0 = dot4(cv, ld4(b0 + n), s0);
            s1 = dot4(cv, ld4(b1 + n), s1);
            s2 = dot4(cv, ld4(b2 + n), s2);
            s3 = dot4(cv, ld4(b3 + n), s3);
        }
        const float *x0 = X + (size_t)min(c0, nrows - 1) * ldp, *x1 = X + (size_t)min(c0 + 1, nrows - 1) * ldp;
        const float *x2 = X + (size_t)min(c0 + 2, nrows - 1) * ldp, *x3 = X + (size_t)min(c0 + 3, nrows - 1) * ldp;
        float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
        for (int p = 0; p < Pp; p += 4) {
            const float4 dv = ld4(dp + p);
            v0 = dot4(dv, ld4(x0 + p), v0);
            v1 = dot4(dv, ld4(x1 + p), v1);
            v2 = dot4(dv, ld4(x2 + p), v2);
            v3 = dot4(dv, ld4(x3 + p), v3);
        }
        if (rr < nrows) {
            const int tr = rr / R;
            const bool k0 = c0 < nrows && c0 / R <= tr, k1 = c0 + 1 < nrows && (c0 + 1) / R <= tr;
            const bool k2 = c0 + 2 < nrows && (c0 + 2) / R <= tr, k3 = c0 + 3 < nrows && (c0 + 3) / R <= tr;
            st4(S + (size_t)rr * ldq + c0, make_float4(k0 ? s0 : 0.f, k1 ? s1 : 0.f, k2 ? s2 : 0.f, k3 ? s3 : 0.f));
            st4(V + (size_t)rr * ldq + c0, make_float4(k0 ? v0 : 0.f, k1 ? v1 : 0.f, k2 ? v2 : 0.f, k3 ? v3 : 0.f));
        }
    }
}

// global (N, P) row-major  <->  shared transposed (P, ldn)
__device__ void load_state_T(float *St, int lds, const float *g, int N, int P, float scale = 1.f,
                             const float *g2 = nullptr, float s2 = 0.f) {
    for (int k = threadIdx.x; k < N * P; k += blockDim.x) {
        const int n = k / P, p = k % P;
        float v = g ? scale * g[k] : 0.f;
        if (g2) v += s2 * g2[k];
        St[(size_t)p * lds + n] = v;
    }
}

// 4-byte asynchronous global -> shared copies (all of a chunk's raw inputs in
// flight at once, instead of one dependent load per loop iteration)
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}
// rows of `words` 4-byte words: dst row k <- src + off(k)
template <typename F>
__device__ __forceinline__ void stage_rows(void *dst, int nrows, int words, F src_row) {
    for (int it = threadIdx.x; it < nrows * words; it += blockDim.x) {
        const int k = it / words, w = it % words;
        cp_async4(static_cast<char *>(dst) + ((size_t)k * words + w) * 4,
                  reinterpret_cast<const char *>(src_row(k)) + (size_t)w * 4);
    }
}

// Chunk preparation shared by the state and the reverse pass: per-token
// coefficients, angles from phi_in, QkNorm inverse RMS, rotated B (and C),
// X = W_x x (and Dy = W_y dy).  The chunk's raw B, C, x, dy and theta are
// first staged in arrays that are free until the prep ends (dBbar, dCbar,
// BG, CG, GP).  Ends with a __syncthreads.
template <typename T>
__device__ void bwd_prep(const BwdArgs &a, const BwdSmem &s, const BwdLayout &Lo, int64_t b, int64_t h,
                         int64_t hg, int64_t t0, int L, const float *phi_in, bool full) {
    const int64_t Tn = a.T, H = a.H, G = a.G;
    const int P = (int)a.P, N = (int)a.N, R = (int)a.R, K = (int)a.K, Q = Lo.Q, ldn = Lo.ldn, ldp = Lo.ldp;
    const int LR = L * R;
    const int tid = threadIdx.x, nt = blockDim.x, warp = tid >> 5, l32 = tid & 31, nw = nt >> 5;
    const T *Bg = static_cast<const T *>(a.B);
    const T *Cg = static_cast<const T *>(a.C);
    const T *x = static_cast<const T *>(a.x);
    const T *dy = static_cast<const T *>(a.dy);
    const float Ah = a.A[h];
    float *dts = s.tk(TK_DT, Q), *lam = s.tk(TK_LAM, Q), *la = s.tk(TK_LA, Q), *cum = s.tk(TK_CUM, Q);
    float *gam = s.tk(TK_GAM, Q), *w = s.tk(TK_W, Q), *ec = s.tk(TK_EC, Q), *cs = s.tk(TK_CS, Q);
    float *cw = s.tk(TK_CW, Q);
    T *sB = reinterpret_cast<T *>(s.dBb), *sC = reinterpret_cast<T *>(s.dCb);
    T *sx = reinterpret_cast<T *>(s.BG), *sdy = reinterpret_cast<T *>(s.CG);
    float *sth = s.GP;
    {
        const int wbc = N * (int)sizeof(T) / 4;   // N is even: whole 4-byte words
        auto brow = [&](int k) { return Bg + (((b * Tn + t0 + k / R) * G + hg) * R + k % R) * N; };
        auto crow = [&](int k) { return Cg + (((b * Tn + t0 + k / R) * G + hg) * R + k % R) * N; };
        stage_rows(sB, LR, wbc, brow);
        if (full) stage_rows(sC, LR, wbc, crow);
        stage_rows(sth, L, K, [&](int k) { return a.theta + ((b * Tn + t0 + k) * H + h) * K; });
        if ((P * (int)sizeof(T)) % 4 == 0) {
            const int wx = P * (int)sizeof(T) / 4;
            stage_rows(sx, L, wx, [&](int k) { return x + ((b * Tn + t0 + k) * H + h) * P; });
            if (full) stage_rows(sdy, L, wx, [&](int k) { return dy + ((b * Tn + t0 + k) * H + h) * P; });
        } else {   // rows not a whole number of words: plain copies
            for (int it = tid; it < L * P; it += nt) {
                const int64_t xi = ((b * Tn + t0 + it / P) * H + h) * P + it % P;
                sx[it] = x[xi];
                if (full) sdy[it] = dy[xi];
            }
        }
        cp_async_wait_all();
    }
    for (int i = tid; i < L; i += nt) {
        const int64_t bt = (b * Tn + t0 + i) * H + h;
        const float dl = a.dt[bt], lm = a.lam[bt];
        float sg = 0.f;
        if (t0 + i + 1 < Tn) sg = (1.f - a.lam[bt + H]) * a.dt[bt + H];
        dts[i] = dl;
        lam[i] = lm;
        la[i] = dl * Ah;
        gam[i] = lm * dl;
        w[i] = lm * dl + sg;
    }
    __syncthreads();   // the staged rows are visible to every thread
    const bool has_norm = a.nrm.wB || a.nrm.wC;
    if (has_norm) {
        for (int row = warp; row < LR; row += nw) {
            float sb = 0.f, sc = 0.f;
            for (int n = l32; n < N; n += 32) {
                const float vb = ldf(sB, row * N + n), vc = full ? ldf(sC, row * N + n) : 0.f;
                sb += vb * vb;
                sc += vc * vc;
            }
            for (int o = 16; o > 0; o >>= 1) {
                sb += __shfl_xor_sync(0xffffffffu, sb, o);
                sc += __shfl_xor_sync(0xffffffffu, sc, o);
            }
            if (l32 == 0) {
                s.inv[row] = rsqrtf(sb / N + a.nrm.eps);
                s.inv[Q * R + row] = rsqrtf(sc / N + a.nrm.eps);
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        float run = 0.f;
        for (int i = 0; i < L; i++) {
            run += la[i];
            cum[i] = run;
        }
    }
    // angles: the running sum of dt theta from the chunk's entering angle
    for (int j = tid; j < K; j += nt) {
        float c = phi_in[j];
        for (int i = 0; i < L; i++) {
            c += dts[i] * sth[i * K + j];
            s.Ph[i * K + j] = c;
        }
    }
    __syncthreads();
    for (int i = tid; i < L; i += nt) {
        ec[i] = expf(cum[i]);
        cs[i] = expf(cum[L - 1] - cum[i]);
        cw[i] = cs[i] * w[i];
    }
    for (int it = tid; it < LR * (N / 2); it += nt) {
        const int j = it % (N / 2), row = it / (N / 2), i = row / R, r = row % R;
        const int base = row * N + 2 * j;
        float b0 = ldf(sB, base), b1 = ldf(sB, base + 1);
        float c0 = full ? ldf(sC, base) : 0.f, c1 = full ? ldf(sC, base + 1) : 0.f;
        if (a.nrm.wB) { b0 *= s.inv[row] * a.nrm.wB[2 * j]; b1 *= s.inv[row] * a.nrm.wB[2 * j + 1]; }
        if (a.nrm.wC) { c0 *= s.inv[Q * R + row] * a.nrm.wC[2 * j]; c1 *= s.inv[Q * R + row] * a.nrm.wC[2 * j + 1]; }
        const int64_t bo = (h * R + r) * N + 2 * j;
        if (a.nrm.biasB) { b0 += a.nrm.biasB[bo]; b1 += a.nrm.biasB[bo + 1]; }
        if (a.nrm.biasC) { c0 += a.nrm.biasC[bo]; c1 += a.nrm.biasC[bo + 1]; }
        float sn = 0.f, cn = 1.f;
        if (j < K) sincosf(s.Ph[i * K + j], &sn, &cn);
        s.Bb[row * ldn + 2 * j] = cn * b0 - sn * b1;
        s.Bb[row * ldn + 2 * j + 1] = sn * b0 + cn * b1;
        if (full) {
            s.Cb[row * ldn + 2 * j] = cn * c0 - sn * c1;
            s.Cb[row * ldn + 2 * j + 1] = sn * c0 + cn * c1;
        }
    }
    for (int it = tid; it < LR * P; it += nt) {
        const int p = it % P, row = it / P, i = row / R, r = row % R;
        s.X[row * ldp + p] = (a.Wx ? a.Wx[(h * R + r) * P + p] : 1.f) * ldf(sx, i * P + p);
        if (full) s.Dy[row * ldp + p] = (a.Wy ? a.Wy[(h * R + r) * P + p] : 1.f) * ldf(sdy, i * P + p);
    }
    __syncthreads();
}

__device__ void zero_smem(float *sm, size_t n) {
    for (size_t k = threadIdx.x; k < n; k += blockDim.x) sm[k] = 0.f;
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Forward state pass: g_in and the entering angle of every chunk.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256, 1) k_bwd_state(BwdArgs a) {
    const int64_t lane = blockIdx.x, b = lane / a.H, h = lane % a.H, hg = h / (a.H / a.G);
    const int64_t Tn = a.T;
    const int P = (int)a.P, N = (int)a.N, R = (int)a.R, K = (int)a.K, Q = a.Q;
    const int64_t NP = (int64_t)N * P, nch = (Tn + Q - 1) / Q;
    const BwdLayout Lo = bwd_layout(P, N, R, K, Q);
    extern __shared__ float sm[];
    const BwdSmem s(sm, Lo);
    const int tid = threadIdx.x, nt = blockDim.x;
    zero_smem(sm, Lo.total);
    float *phi = s.misc;   // K: running angle
    for (int j = tid; j < K; j += nt) phi[j] = a.angle0 ? a.angle0[lane * K + j] : 0.f;
    float f0 = 0.f;
    if (Tn > 0) {
        const int64_t i0 = (b * Tn) * a.H + h;
        f0 = (1.f - a.lam[i0]) * a.dt[i0];
    }
    load_state_T(s.gs, Lo.ldn, a.h0 ? a.h0 + lane * NP : nullptr, N, P, 1.f,
                 a.prevBx0 ? a.prevBx0 + lane * NP : nullptr, f0);
    __syncthreads();
    float *slot0 = a.ws + a.ws_slots + (size_t)lane * nch * (NP + K);
    for (int64_t c = 0; c < nch; c++) {
        const int64_t t0 = c * Q;
        const int L = (int)((Tn - t0) < Q ? (Tn - t0) : Q);
        float *slot = slot0 + (size_t)c * (NP + K);
        for (int64_t k = tid; k < NP; k += nt) slot[k] = s.gs[(size_t)(k % P) * Lo.ldn + k / P];
        for (int j = tid; j < K; j += nt) slot[NP + j] = phi[j];
        bwd_prep<T>(a, s, Lo, b, h, hg, t0, L, phi, false);
        // g_out = e^{cum_end} g_in + sum_t e^{cum_end-cum_t} w_t Bbar_t X_t^T
        mm_state_update(s.gs, Lo.ldn, Lo.Np, P, s.tk(TK_EC, Q)[L - 1], s.Bb, Lo.ldn, s.X, Lo.ldp, s.tk(TK_CW, Q), R,
                        L * R);
        for (int j = tid; j < K; j += nt) phi[j] = s.Ph[(L - 1) * K + j];
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Reverse pass.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256, 1) k_bwd_chunks(BwdArgs a) {
    const int64_t lane = blockIdx.x, b = lane / a.H, h = lane % a.H, hg = h / (a.H / a.G);
    const int64_t Tn = a.T, H = a.H;
    const int P = (int)a.P, N = (int)a.N, R = (int)a.R, K = (int)a.K, Q = a.Q;
    const int64_t NP = (int64_t)N * P, nch = (Tn + Q - 1) / Q;
    const int RP = R * P, RN = R * N;
    const BwdLayout Lo = bwd_layout(P, N, R, K, Q);
    const int ldn = Lo.ldn, ldp = Lo.ldp, Np = Lo.Np, ldq = Lo.ldq;
    extern __shared__ float sm[];
    const BwdSmem s(sm, Lo);
    const int tid = threadIdx.x, nt = blockDim.x, warp = tid >> 5, l32 = tid & 31, nw = nt >> 5;
    const T *Bg = static_cast<const T *>(a.B);
    const T *Cg = static_cast<const T *>(a.C);
    const T *x = static_cast<const T *>(a.x);
    const T *dy = static_cast<const T *>(a.dy);
    const float Ah = a.A[h], Dh = a.D[h];
    float *Gphi = s.misc;                // K: angle adjoint flowing backwards
    float *pend = s.misc + 2 * K + 32;   // [0] ddt, [1] dlam of the pending token
    float *par = s.par;
    const ParOff po(P, N, R);
    const size_t oWy = po.Wy, owB = po.wB, owC = po.wC, obB = po.bB, obC = po.bC;

    zero_smem(sm, Lo.total);
    load_state_T(s.Gs, ldn, a.dh ? a.dh + lane * NP : nullptr, N, P);
    for (int j = tid; j < K; j += nt) Gphi[j] = a.da ? a.da[lane * K + j] : 0.f;
    __syncthreads();
    const float *slot0 = a.ws + a.ws_slots + (size_t)lane * nch * (NP + K);
    float *dBout = a.G < a.H ? a.ws + a.ws_dBh : a.dB;
    float *dCout = a.G < a.H ? a.ws + a.ws_dCh : a.dC;
    // B/C gradient rows: per head (workspace, summed over the group later) or the group row itself
    auto grad_row = [&](int64_t t, int r) -> int64_t {
        return a.G < a.H ? (((b * Tn + t) * H + h) * R + r) * N : (((b * Tn + t) * a.G + hg) * R + r) * N;
    };

    for (int64_t c = nch - 1; c >= 0; c--) {
        const int64_t t0 = c * Q;
        const int L = (int)((Tn - t0) < Q ? (Tn - t0) : Q);
        const int LR = L * R;
        const bool last = (c == nch - 1);
        const float *slot = slot0 + (size_t)c * (NP + K);
        load_state_T(s.gs, ldn, slot, N, P);
        bwd_prep<T>(a, s, Lo, b, h, hg, t0, L, slot + NP, true);
        const float *dts = s.tk(TK_DT, Q), *lam = s.tk(TK_LAM, Q), *cum = s.tk(TK_CUM, Q);
        const float *gam = s.tk(TK_GAM, Q), *w = s.tk(TK_W, Q), *ec = s.tk(TK_EC, Q), *cs = s.tk(TK_CS, Q);
        float *q = s.tk(TK_Q, Q), *yi = s.tk(TK_YI, Q), *dcum = s.tk(TK_DCUM, Q), *dw = s.tk(TK_DW, Q);
        float *dla = s.tk(TK_DLA, Q), *dth = s.tk(TK_DTH, Q), *dyx = s.tk(TK_DYX, Q), *dgam = s.tk(TK_DGAM, Q);

        // the causal mask M[s,t] (t <= s), zero above the diagonal
        for (int it = tid; it < L * L; it += nt) {
            const int tt = it % L, ss = it / L;
            s.MK[ss * Q + tt] = tt < ss ? expf(cum[ss] - cum[tt]) * w[tt] : (tt == ss ? gam[ss] : 0.f);
        }
        // (e) BG = Bbar Gin^T-product (rows x P), CG = Cbar g_in-product; S = Cbar Bbar^T,
        // V = Dy X^T (causal pairs only)
        mm_rows_by_state(s.Bb, ldn, LR, s.Gs, ldn, Np, P, s.BG, ldp);
        mm_rows_by_state(s.Cb, ldn, LR, s.gs, ldn, Np, P, s.CG, ldp);
        scores(s.S, s.V, ldq, s.Cb, s.Bb, ldn, Np, s.Dy, s.X, ldp, Lo.Pp, LR, R);
        __syncthreads();
        // (f) token scalars: q_t = <Gin, U_t>, yi_s = sum_r Dy_s . CG_s, dM, dy . x
        for (int i = warp; i < L; i += nw) {
            float qq = 0.f, yy = 0.f, xx = 0.f;
            for (int k = l32; k < RP; k += 32) {
                const int row = i * R + k / P, p = k % P;
                qq += s.BG[row * ldp + p] * s.X[row * ldp + p];
                yy += s.Dy[row * ldp + p] * s.CG[row * ldp + p];
            }
            for (int p = l32; p < P; p += 32) {
                const int64_t xi = ((b * Tn + t0 + i) * H + h) * P + p;
                xx += ldf(dy, xi) * ldf(x, xi);
            }
            for (int o = 16; o > 0; o >>= 1) {
                qq += __shfl_xor_sync(0xffffffffu, qq, o);
                yy += __shfl_xor_sync(0xffffffffu, yy, o);
                xx += __shfl_xor_sync(0xffffffffu, xx, o);
            }
            if (l32 == 0) { q[i] = qq; yi[i] = yy; dyx[i] = xx; }
        }
        for (int it = tid; it < L * L; it += nt) {
            const int tt = it % L, ss = it / L;
            float v = 0.f;
            if (tt <= ss)
                for (int r2 = 0; r2 < R; r2++)
                    for (int r1 = 0; r1 < R; r1++) {
                        const int rr = ss * R + r2, cr = tt * R + r1;
                        v += s.S[rr * ldq + cr] * s.V[rr * ldq + cr];
                    }
            s.DM[ss * Q + tt] = v;
        }
        float gG;   // <Gin, g_in>
        {
            float v = 0.f;
            for (int k = tid; k < Lo.Pp * ldn; k += nt) v += s.Gs[k] * s.gs[k];
            gG = block_sum(v, s.misc + 2 * K);
        }
        // (h1) the inter parts of dBbar and dCbar: Gin X_t and g_in Dy_s (rows x Np)
        mm_rows_by_stateT(s.X, ldp, LR, s.Gs, ldn, Np, P, s.dBb, ldn);
        mm_rows_by_stateT(s.Dy, ldp, LR, s.gs, ldn, Np, P, s.dCb, ldn);
        __syncthreads();
        // (g) mask, decay and lookahead adjoints per token (M[s,t] = e^{cum_s-cum_t} w_t, t < s)
        for (int i = tid; i < L; i += nt) {
            float dc = ec[i] * yi[i] - cs[i] * w[i] * q[i];
            for (int tt = 0; tt < i; tt++) dc += s.DM[i * Q + tt] * s.MK[i * Q + tt];
            float dwi = cs[i] * q[i];
            for (int ss = i + 1; ss < L; ss++) {
                dc -= s.DM[ss * Q + i] * s.MK[ss * Q + i];
                dwi += s.DM[ss * Q + i] * expf(cum[ss] - cum[i]);
            }
            if (i == L - 1) {
                float st = ec[L - 1] * gG;
                for (int tt = 0; tt < L; tt++) st += cs[tt] * w[tt] * q[tt];
                dc += st;
            }
            dcum[i] = dc;
            dw[i] = dwi;
            dgam[i] = s.DM[i * Q + i] + dwi;
        }
        // the masked scores S <- M o S, V <- M o V (the token mask expanded over ranks)
        for (int it = tid; it < LR * LR; it += nt) {
            const int cr = it % LR, rr = it / LR;
            const float m = s.MK[(rr / R) * Q + cr / R];
            s.S[rr * ldq + cr] *= m;
            s.V[rr * ldq + cr] *= m;
        }
        __syncthreads();
        // (h2) dX = w cs BG + S'^T Dy (into BG); dBbar = w cs GX + V'^T Cbar (into dBb);
        // dCbar = e^{cum} GD + V' Bbar (into dCb); MIMO: Y = e^{cum} CG + S' X (into CG)
        const float *cw = s.tk(TK_CW, Q);
        mm_wT_rows(s.BG, ldp, LR, s.S, ldq, LR, s.Dy, ldp, Lo.Pp, cw, R);
        mm_wT_rows(s.dBb, ldn, LR, s.V, ldq, LR, s.Cb, ldn, Np, cw, R);
        mm_w_rows(s.dCb, ldn, LR, s.V, ldq, LR, s.Bb, ldn, Np, ec, R);
        if (a.dWy) mm_w_rows(s.CG, ldp, LR, s.S, ldq, LR, s.X, ldp, Lo.Pp, ec, R);
        __syncthreads();
        if (last && a.du) {   // prev_Bx_final = U_{T-1}: its adjoint reaches the last token's rows
            const float *du = a.du + lane * NP;
            for (int it = tid; it < R * P; it += nt) {
                const int p = it % P, cr = (L - 1) * R + it / P;
                float e = 0.f;
                for (int n = 0; n < N; n++) e += du[n * P + p] * s.Bb[cr * ldn + n];
                s.BG[cr * ldp + p] += e;
            }
            for (int it = tid; it < R * N; it += nt) {
                const int n = it % N, cr = (L - 1) * R + it / N;
                float e = 0.f;
                for (int p = 0; p < P; p++) e += du[n * P + p] * s.X[cr * ldp + p];
                s.dBb[cr * ldn + n] += e;
            }
            __syncthreads();
        }
        // dx = D dy + sum_r W_x[r] dX_r
        for (int it = tid; it < L * P; it += nt) {
            const int p = it % P, i = it / P;
            const int64_t xi = ((b * Tn + t0 + i) * H + h) * P + p;
            float dxs = Dh * ldf(dy, xi);
            for (int r = 0; r < R; r++) dxs += (a.Wx ? a.Wx[(h * R + r) * P + p] : 1.f) * s.BG[(i * R + r) * ldp + p];
            if (a.dx) a.dx[xi] = dxs;
        }
        if (tid == 0) {
            float run = 0.f;
            for (int i = L - 1; i >= 0; i--) {
                run += dcum[i];
                dla[i] = run;
            }
        }
        if (a.dWy)   // dW_y partial: sum_s dy_s[p] Y_{s,r}[p] (one thread per (r, p))
            for (int it = tid; it < RP; it += nt) {
                const int p = it % P, r = it / P;
                float acc = 0.f;
                for (int i = 0; i < L; i++)
                    acc += ldf(dy, ((b * Tn + t0 + i) * H + h) * P + p) * s.CG[(i * R + r) * ldp + p];
                par[oWy + it] += acc;
            }
        // dW_x partial: sum_t x_t[p] dX_{t,r}[p] (one thread per (r, p))
        for (int it = tid; it < RP; it += nt) {
            const int p = it % P, r = it / P;
            float acc = 0.f;
            for (int i = 0; i < L; i++)
                acc += ldf(x, ((b * Tn + t0 + i) * H + h) * P + p) * s.BG[(i * R + r) * ldp + p];
            par[po.Wx + it] += acc;
        }
        // (i) Gin <- e^{cum_end} Gin + sum_{s,r} e^{cum_s} Cbar_{s,r} Dy_{s,r}^T
        mm_state_update(s.Gs, ldn, Np, P, ec[L - 1], s.Cb, ldn, s.Dy, ldp, ec, R, LR);
        // (j) rotation adjoint: local angle adjoint per (token, pair)
        for (int it = tid; it < L * K; it += nt) {
            const int j = it % K, i = it / K;
            float gp = 0.f;
            for (int r = 0; r < R; r++) {
                const int row = i * R + r;
                const float *bb = s.Bb + row * ldn, *cb = s.Cb + row * ldn;
                const float *db = s.dBb + row * ldn, *dc = s.dCb + row * ldn;
                gp += -db[2 * j] * bb[2 * j + 1] + db[2 * j + 1] * bb[2 * j];
                gp += -dc[2 * j] * cb[2 * j + 1] + dc[2 * j + 1] * cb[2 * j];
            }
            s.GP[i * K + j] = gp;
        }
        __syncthreads();
        // the angle adjoint runs backwards: GPhi_t = local_t + GPhi_{t+1}; dtheta_t = dt_t GPhi_t
        for (int j = tid; j < K; j += nt) {
            float g = Gphi[j];
            for (int i = L - 1; i >= 0; i--) {
                g += s.GP[i * K + j];
                s.GP[i * K + j] = g;
                if (a.dtheta) a.dtheta[((b * Tn + t0 + i) * H + h) * K + j] = dts[i] * g;
            }
            Gphi[j] = g;
        }
        // pair adjoints turned back by -Phi_t (pairs from K on pass through)
        for (int it = tid; it < LR * (N / 2); it += nt) {
            const int j = it % (N / 2), row = it / (N / 2), i = row / R;
            if (j >= K) continue;
            float sn, cn;
            sincosf(s.Ph[i * K + j], &sn, &cn);
            float *db = s.dBb + row * ldn, *dc = s.dCb + row * ldn;
            const float b0 = db[2 * j], b1 = db[2 * j + 1], c0 = dc[2 * j], c1 = dc[2 * j + 1];
            db[2 * j] = cn * b0 + sn * b1;
            db[2 * j + 1] = -sn * b0 + cn * b1;
            dc[2 * j] = cn * c0 + sn * c1;
            dc[2 * j + 1] = -sn * c0 + cn * c1;
        }
        __syncthreads();
        // theta . GPhi per token (its dt adjoint); QkNorm row sums
        for (int i = warp; i < L; i += nw) {
            float v = 0.f;
            for (int j = l32; j < K; j += 32) v += a.theta[((b * Tn + t0 + i) * H + h) * K + j] * s.GP[i * K + j];
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (l32 == 0) dth[i] = v;
        }
        if (a.nrm.wB || a.nrm.wC) {
            for (int row = warp; row < LR; row += nw) {
                const int64_t base = (((b * Tn + t0 + row / R) * a.G + hg) * R + row % R) * N;
                float sb = 0.f, sc = 0.f;
                for (int n = l32; n < N; n += 32) {
                    if (a.nrm.wB) sb += s.dBb[row * ldn + n] * a.nrm.wB[n] * ldf(Bg, base + n);
                    if (a.nrm.wC) sc += s.dCb[row * ldn + n] * a.nrm.wC[n] * ldf(Cg, base + n);
                }
                for (int o = 16; o > 0; o >>= 1) {
                    sb += __shfl_xor_sync(0xffffffffu, sb, o);
                    sc += __shfl_xor_sync(0xffffffffu, sc, o);
                }
                if (l32 == 0) { s.rsc[row] = sb; s.rsc[Q * R + row] = sc; }
            }
        }
        __syncthreads();
        // gain and bias partials (fixed thread-to-element map: deterministic)
        if (a.nrm.wB || a.nrm.wC)
            for (int n = tid; n < N; n += nt) {
                float gb = 0.f, gc = 0.f;
                for (int row = 0; row < LR; row++) {
                    const int64_t base = (((b * Tn + t0 + row / R) * a.G + hg) * R + row % R) * N;
                    if (a.nrm.wB) gb += s.dBb[row * ldn + n] * ldf(Bg, base + n) * s.inv[row];
                    if (a.nrm.wC) gc += s.dCb[row * ldn + n] * ldf(Cg, base + n) * s.inv[Q * R + row];
                }
                par[owB + n] += gb;
                par[owC + n] += gc;
            }
        if (a.nrm.biasB || a.nrm.biasC)
            for (int k = tid; k < RN; k += nt) {
                const int n = k % N, r = k / N;
                float gb = 0.f, gc = 0.f;
                for (int i = 0; i < L; i++) {
                    gb += s.dBb[(i * R + r) * ldn + n];
                    gc += s.dCb[(i * R + r) * ldn + n];
                }
                par[obB + k] += gb;
                par[obC + k] += gc;
            }
        // raw B/C adjoints: through the QkNorm (when on)
        for (int it = tid; it < LR * N; it += nt) {
            const int n = it % N, row = it / N, i = row / R, r = row % R;
            const int64_t base = (((b * Tn + t0 + i) * a.G + hg) * R + r) * N;
            float gb = s.dBb[row * ldn + n], gc = s.dCb[row * ldn + n];
            if (a.nrm.wB) {
                const float iv = s.inv[row];
                gb = iv * gb * a.nrm.wB[n] - ldf(Bg, base + n) * iv * iv * iv * s.rsc[row] / N;
            }
            if (a.nrm.wC) {
                const float iv = s.inv[Q * R + row];
                gc = iv * gc * a.nrm.wC[n] - ldf(Cg, base + n) * iv * iv * iv * s.rsc[Q * R + row] / N;
            }
            const int64_t o = grad_row(t0 + i, r) + n;
            if (dBout) dBout[o] = gb;
            if (dCout) dCout[o] = gc;
        }
        // (k) dt and lam adjoints; the first token waits for dw of the token before it
        if (tid == 0) {
            float dAl = 0.f, dDl = 0.f;
            for (int i = L - 1; i >= 0; i--) {
                const int64_t bt = (b * Tn + t0 + i) * H + h;
                float ddt = dla[i] * Ah + dgam[i] * lam[i] + dth[i];
                float dlm = dgam[i] * dts[i];
                if (i > 0) {
                    ddt += dw[i - 1] * (1.f - lam[i]);
                    dlm -= dw[i - 1] * dts[i];
                    if (a.ddt) a.ddt[bt] = ddt;
                    if (a.dlam) a.dlam[bt] = dlm;
                } else {
                    if (!last) {   // finish the pending first token of the chunk after this one
                        const int64_t bn = bt + (int64_t)L * H;
                        const float ln = a.lam[bn], dn = a.dt[bn];
                        if (a.ddt) a.ddt[bn] = pend[0] + dw[L - 1] * (1.f - ln);
                        if (a.dlam) a.dlam[bn] = pend[1] - dw[L - 1] * dn;
                    }
                    pend[0] = ddt;
                    pend[1] = dlm;
                }
                dAl += dla[i] * dts[i];
                dDl += dyx[i];
            }
            par[0] += dAl;
            par[1] += dDl;
        }
        __syncthreads();
    }
    // the initial state: g_{-1} = h0 + f0 prev_Bx0, f0 = (1-lam_0) dt_0
    float f0 = 0.f, dwm = 0.f;
    if (Tn > 0) {
        const int64_t i0 = (b * Tn) * H + h;
        f0 = (1.f - a.lam[i0]) * a.dt[i0];
        float v = 0.f;
        if (a.prevBx0)
            for (int64_t k = tid; k < NP; k += nt) v += s.Gs[(size_t)(k % P) * ldn + k / P] * a.prevBx0[lane * NP + k];
        dwm = block_sum(v, s.misc + 2 * K);
        if (tid == 0) {
            if (a.ddt) a.ddt[i0] = pend[0] + dwm * (1.f - a.lam[i0]);
            if (a.dlam) a.dlam[i0] = pend[1] - dwm * a.dt[i0];
        }
    }
    for (int64_t k = tid; k < NP; k += nt) {
        const float g = s.Gs[(size_t)(k % P) * ldn + k / P];
        if (a.dh0) a.dh0[lane * NP + k] = g;
        // with no token, prev_Bx_final is prev_Bx0 itself
        if (a.du0) a.du0[lane * NP + k] = Tn > 0 ? f0 * g : (a.du ? a.du[lane * NP + k] : 0.f);
    }
    for (int j = tid; j < K; j += nt)
        if (a.da0) a.da0[lane * K + j] = Gphi[j];
    __syncthreads();
    float *pout = a.ws + a.ws_partial + (size_t)lane * par_floats(P, N, R);
    for (int k = tid; k < (int)par_floats(P, N, R); k += nt) pout[k] = par[k];
}

// ---------------------------------------------------------------------------
// Shared parameters: sum the per-lane partials over the batch (and over all
// lanes for the gains); grouped B/C: sum the heads of each group.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bwd_params(BwdArgs a) {
    const int64_t P = a.P, N = a.N, R = a.R, H = a.H, RP = R * P, RN = R * N;
    const size_t pf = par_floats(P, N, R);
    const float *part = a.ws + a.ws_partial;
    const ParOff po(P, N, R);
    const size_t owB = po.wB, owC = po.wC, obB = po.bB, obC = po.bC;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, gstride = (int64_t)gridDim.x * blockDim.x;
    // per head: A, D, W_x, W_y, biases
    const int64_t per_head = 2 + 2 * RP + 2 * RN;
    for (int64_t it = gtid; it < H * per_head; it += gstride) {
        const int64_t h = it / per_head, k = it % per_head;
        size_t off;
        float *dst;
        if (k == 0) { off = 0; dst = a.dA ? a.dA + h : nullptr; }
        else if (k == 1) { off = 1; dst = a.dD ? a.dD + h : nullptr; }
        else if (k < 2 + RP) { off = po.Wx + (k - 2); dst = a.dWx ? a.dWx + h * RP + (k - 2) : nullptr; }
        else if (k < 2 + 2 * RP) { off = po.Wy + (k - 2 - RP); dst = a.dWy ? a.dWy + h * RP + (k - 2 - RP) : nullptr; }
        else if (k < 2 + 2 * RP + RN) { off = obB + (k - 2 - 2 * RP); dst = a.dbB ? a.dbB + h * RN + (k - 2 - 2 * RP) : nullptr; }
        else { off = obC + (k - 2 - 2 * RP - RN); dst = a.dbC ? a.dbC + h * RN + (k - 2 - 2 * RP - RN) : nullptr; }
        if (!dst) continue;
        float acc = 0.f;
        for (int64_t b = 0; b < a.Bt; b++) acc += part[(size_t)(b * H + h) * pf + off];
        *dst = acc;
    }
    // gains: every lane
    for (int64_t it = gtid; it < 2 * N; it += gstride) {
        const int64_t n = it % N;
        const bool isC = it >= N;
        float *dst = isC ? a.dwC : a.dwB;
        if (!dst) continue;
        float acc = 0.f;
        for (int64_t l = 0; l < a.Bt * H; l++) acc += part[(size_t)l * pf + (isC ? owC : owB) + n];
        dst[n] = acc;
    }
    // grouped B/C: sum the per-head rows of each group in head order
    if (a.G < a.H) {
        const int64_t hpg = H / a.G, rows = a.Bt * a.T * a.G * RN;
        const float *dBh = a.ws + a.ws_dBh, *dCh = a.ws + a.ws_dCh;
        for (int64_t it = gtid; it < rows; it += gstride) {
            const int64_t e = it % RN, bt = it / RN / a.G, g = (it / RN) % a.G;
            float sb = 0.f, sc = 0.f;
            for (int64_t k = 0; k < hpg; k++) {
                const int64_t src = (bt * H + g * hpg + k) * RN + e;
                sb += dBh[src];
                sc += dCh[src];
            }
            if (a.dB) a.dB[it] = sb;
            if (a.dC) a.dC[it] = sc;
        }
    }
}

template <typename T>
static cudaError_t launch_bwd_t(BwdArgs a, cudaStream_t st) {
    const int64_t lanes = a.Bt * a.H;
    const BwdWs w = bwd_ws(a, a.Q);
    a.ws_slots = w.slots;
    a.ws_partial = w.partial;
    a.ws_dBh = w.dBh;
    a.ws_dCh = w.dCh;
    const size_t smem = sizeof(float) * bwd_layout(a.P, a.N, a.R, a.K, a.Q).total;
    cudaError_t e;
    cudaFuncSetAttribute(k_bwd_state<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_bwd_chunks<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (a.T > 0) {
        k_bwd_state<T><<<(unsigned)lanes, 256, smem, st>>>(a);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    k_bwd_chunks<T><<<(unsigned)lanes, 256, smem, st>>>(a);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_params<<<148, 256, 0, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_scan_bwd(const BwdArgs &a, m3_dtype dt, cudaStream_t s) {
    if (a.Bt * a.H == 0) return cudaSuccess;
    return dt == M3_BF16 ? launch_bwd_t<__nv_bfloat16>(a, s) : launch_bwd_t<float>(a, s);
}

}  // namespace m3
