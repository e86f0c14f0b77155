/*
 * m3_oracle.c -- fp64 CPU oracle for the Mamba-3 selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * definition that the CUDA library is checked against.  Only the tests,
 * the package's smoke check and the benchmark's CPU-baseline leg may load
 * it.  It shares no code, header, table or helper with the CUDA path.
 *
 * Sources (the pages this restates, by title and section):
 *   [dotLLM]  "Mamba-3 (real algorithm) kernel-level PoC" pull request,
 *             sections "Stage A" (Discretize, QkNorm, DataRoPE, MimoProject,
 *             SelectiveScan -- trapezoidal scan, Eq. 9, with a prev_Bx second
 *             state), "Key findings" (lambda and theta are per token; BC-bias
 *             after QkNorm, before RoPE), the streaming-decode comment
 *             (shifted_gamma[t] = DT[t+1](1-trap[t+1]), scale = gamma +
 *             shifted_gamma; boundary fold DT[0](1-trap[0]) applied before the
 *             scan's alpha) and "Mamba-3 MIMO streaming decode" (state is
 *             rank-summed; cum_angle is rank-free).
 *   [torchmamba] "TorchMamba" README, sections "Models" (3-term trap
 *             h = a h + b B_{-1} x_{-1} + g B x; MIMO = rank-R update on a
 *             shared (N,P) state), "Math notes" (Prop. 1 Eqs. 5-6, Eq. 7
 *             L = 1SS @ band, Props. 2-4 data-dependent pairwise rotations,
 *             App. C per-head expand/contract vectors) and "Behavioral notes"
 *             (RoPE needs even N; states never below fp32).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   alpha_t = exp(dt_t A_h), beta_t = (1-lam_t) dt_t alpha_t,
 *   gamma_t = lam_t dt_t;  per-step angle dt_t * theta_t;  adjacent pairs
 *   (2i, 2i+1) rotated by +Phi;  all N/2 pairs rotate;  h0 = prev_Bx0 = 0 and
 *   Phi0 = 0 unless given;  MIMO expand/contract vectors W_x, W_y of shape
 *   (H,R,P);  QkNorm gain of shape (N), bias of shape (H,R,N).
 *
 * Layouts (row-major, last index fastest):
 *   x, y (Bt,T,H,P); dt, lam (Bt,T,H); A, D (H); theta (Bt,T,H,K);
 *   B, C (Bt,T,G,R,N) with R = 1 for SISO (G = H unless grouped);
 *   W_x, W_y (H,R,P); h, prev_Bx (Bt,H,N,P); angle (Bt,H,K);
 *   K = N/2 unless partial RoPE.
 *
 * Every function returns 0 on success, -1 on a bad argument.
 */
#include <math.h>
#include <pthread.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Host allocation that never returns NULL: the oracle is a checker, so
 * running out of memory ends the process loudly instead of yielding a
 * partial result. */
static void *xmalloc(size_t n)
{
    void *p = malloc(n ? n : 1);
    if (!p) {
        fputs("m3_oracle: out of host memory\n", stderr);
        abort();
    }
    return p;
}

typedef struct {
    long batch, seqlen, nheads, headdim, dstate, rank;
    long ngroups;    /* B/C groups G (H % G == 0); 0 means G = H            */
    long rope_pairs; /* pairs (2i, 2i+1), i < K, that rotate; 0 means N/2  */
} m3o_dims;

/* Grouped B/C (torchmamba "Models": n_groups, H % G == 0) and partial RoPE
 * (dotLLM pull request, real-checkpoint run: num_rope_angles = 32 of
 * d_state 128, rope_fraction 0.5).  Head h reads the B/C row of group
 * h / (H / G); only the first K pairs rotate (theta and the angle then hold K
 * values per head), the others pass through unrotated. */
static long n_groups(m3o_dims d) { return d.ngroups > 0 ? d.ngroups : d.nheads; }
static long n_pairs(m3o_dims d) { return d.rope_pairs > 0 ? d.rope_pairs : d.dstate / 2; }
/* offset of the B/C row (rank r) read by head h at (b, t) */
static long bc_off(m3o_dims d, long b, long t, long h, long r)
{
    long G = n_groups(d), R = d.rank < 1 ? 1 : d.rank;
    return (((b * d.seqlen + t) * G + h / (d.nheads / G)) * R + r) * d.dstate;
}

typedef struct {
    const double *normw_B, *normw_C; /* (N) or NULL: QkNorm off          */
    const double *bias_B, *bias_C;   /* (H,R,N) or NULL: bias off         */
    double eps;                      /* RMSNorm epsilon                   */
} m3o_bcnorm;

/* ------------------------------------------------------------------------ */
/* S1: trapezoidal discretization (dotLLM "Stage A: Mamba3Discretize";      */
/* torchmamba "Math notes", Prop. 1).                                        */
/* ------------------------------------------------------------------------ */
int m3o_discretize(const double *dt, const double *A, const double *lam,
                   long Bt, long T, long H,
                   double *alpha, double *beta, double *gamma)
{
    if (!dt || !A || !lam || !alpha || !beta || !gamma) return -1;
    for (long b = 0; b < Bt; b++)
        for (long t = 0; t < T; t++)
            for (long h = 0; h < H; h++) {
                long i = (b * T + t) * H + h;
                double a = exp(dt[i] * A[h]);
                alpha[i] = a;
                beta[i] = (1.0 - lam[i]) * dt[i] * a;
                gamma[i] = lam[i] * dt[i];
            }
    return 0;
}

/* QkNorm (RMSNorm over N, gain w) then per-head bias; dotLLM "Key findings":
 * the bias is added after the norm and before the rotation. */
static void bc_prepare(const double *src, long N, const double *w,
                       const double *bias, double eps, double *dst)
{
    if (w) {
        double ss = 0.0;
        for (long n = 0; n < N; n++) ss += src[n] * src[n];
        double inv = 1.0 / sqrt(ss / (double)N + eps);
        for (long n = 0; n < N; n++) dst[n] = src[n] * inv * w[n];
    } else {
        for (long n = 0; n < N; n++) dst[n] = src[n];
    }
    if (bias)
        for (long n = 0; n < N; n++) dst[n] += bias[n];
}

/* Rotate adjacent pairs (2i, 2i+1), i < K, of v by the angles phi[i]; the
 * remaining elements pass through. */
static void rotate_pairs(const double *v, const double *phi, long K, long N, double *out)
{
    for (long i = 0; i < K; i++) {
        double c = cos(phi[i]), s = sin(phi[i]);
        double v0 = v[2 * i], v1 = v[2 * i + 1];
        out[2 * i] = c * v0 - s * v1;
        out[2 * i + 1] = s * v0 + c * v1;
    }
    for (long n = 2 * K; n < N; n++) out[n] = v[n];
}

/* ------------------------------------------------------------------------ */
/* S2: QkNorm + BC-bias + data-dependent RoPE (dotLLM "Stage A:             */
/* Mamba3QkNorm / Mamba3DataRoPE"; torchmamba "Math notes", Props. 2-4).    */
/* Phi_t = Phi_{t-1} + dt_t * theta_t (per pair), B_rot = R(Phi_t) B.        */
/* ------------------------------------------------------------------------ */
int m3o_rope_bc(const double *B, const double *C, const double *theta,
                const double *dt, const double *angle0, const m3o_bcnorm *nrm,
                m3o_dims d, double *B_rot, double *C_rot, double *angle_final)
{
    long Bt = d.batch, T = d.seqlen, H = d.nheads, N = d.dstate;
    long R = d.rank < 1 ? 1 : d.rank;
    if (!B || !C || !theta || !dt || !B_rot || !C_rot) return -1;
    if (N <= 0 || (N & 1)) return -1;
    long G = n_groups(d), K = n_pairs(d);
    if (H % G || K < 1 || K > N / 2) return -1;
    double *phi = (double *)xmalloc(sizeof(double) * K);
    double *tmp = (double *)xmalloc(sizeof(double) * N);
    for (long b = 0; b < Bt; b++)
        for (long h = 0; h < H; h++) {
            for (long i = 0; i < K; i++)
                phi[i] = angle0 ? angle0[(b * H + h) * K + i] : 0.0;
            for (long t = 0; t < T; t++) {
                long bth = (b * T + t) * H + h;
                for (long i = 0; i < K; i++)
                    phi[i] += dt[bth] * theta[bth * K + i];
                for (long r = 0; r < R; r++) {
                    long off = (bth * R + r) * N;          /* per-head output row */
                    long offin = bc_off(d, b, t, h, r);    /* the group's input row */
                    const double *bb = nrm && nrm->bias_B ? nrm->bias_B + (h * R + r) * N : NULL;
                    const double *cb = nrm && nrm->bias_C ? nrm->bias_C + (h * R + r) * N : NULL;
                    bc_prepare(B + offin, N, nrm ? nrm->normw_B : NULL, bb, nrm ? nrm->eps : 0.0, tmp);
                    rotate_pairs(tmp, phi, K, N, B_rot + off);
                    bc_prepare(C + offin, N, nrm ? nrm->normw_C : NULL, cb, nrm ? nrm->eps : 0.0, tmp);
                    rotate_pairs(tmp, phi, K, N, C_rot + off);
                }
            }
            if (angle_final)
                for (long i = 0; i < K; i++)
                    angle_final[(b * H + h) * K + i] = phi[i];
        }
    free(phi);
    free(tmp);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Lane workers.  The (b,h) lanes are independent; each worker walks its    */
/* lanes in order and each lane sequentially over t.                         */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *x, *dt, *A, *lam, *theta, *B, *C, *D, *Wx, *Wy;
    const m3o_bcnorm *nrm;
    const double *h0, *prevBx0, *angle0;
    m3o_dims d;
    double *y, *h_out, *prevBx_out, *angle_out;
    long chunk;       /* only for the chunked self-test variant */
    long lane_begin, lane_end;
    int kind;         /* 0 = SISO loop, 1 = MIMO loop, 2 = SISO chunked */
} lane_job;

/* SISO recurrence for one lane (dotLLM "Mamba3SelectiveScan", Eq. 9):
 *   U_t   = B_rot_t x_t^T                      (N x P)
 *   h_t   = alpha_t h_{t-1} + beta_t U_{t-1} + gamma_t U_t
 *   y_t   = C_rot_t^T h_t + D_h x_t
 * with h_{-1} = h0 and U_{-1} = prev_Bx0. */
static void siso_lane(const lane_job *J, long b, long h)
{
    long T = J->d.seqlen, H = J->d.nheads, P = J->d.headdim, N = J->d.dstate;
    long NP = N * P;
    double *hs = (double *)xmalloc(sizeof(double) * NP);
    double *Up = (double *)xmalloc(sizeof(double) * NP);
    long K = n_pairs(J->d);
    double *phi = (double *)xmalloc(sizeof(double) * K);
    double *tmp = (double *)xmalloc(sizeof(double) * N);
    double *Bb = (double *)xmalloc(sizeof(double) * N);
    double *Cb = (double *)xmalloc(sizeof(double) * N);
    long lane = b * H + h;
    for (long k = 0; k < NP; k++) {
        hs[k] = J->h0 ? J->h0[lane * NP + k] : 0.0;
        Up[k] = J->prevBx0 ? J->prevBx0[lane * NP + k] : 0.0;
    }
    for (long i = 0; i < K; i++)
        phi[i] = J->angle0 ? J->angle0[lane * K + i] : 0.0;
    const m3o_bcnorm *nr = J->nrm;
    for (long t = 0; t < T; t++) {
        long bth = (b * T + t) * H + h;
        double dl = J->dt[bth], lm = J->lam[bth];
        double al = exp(dl * J->A[h]);
        double be = (1.0 - lm) * dl * al;
        double ga = lm * dl;
        for (long i = 0; i < K; i++) phi[i] += dl * J->theta[bth * K + i];
        bc_prepare(J->B + bc_off(J->d, b, t, h, 0), N, nr ? nr->normw_B : NULL,
                   nr && nr->bias_B ? nr->bias_B + h * N : NULL, nr ? nr->eps : 0.0, tmp);
        rotate_pairs(tmp, phi, K, N, Bb);
        bc_prepare(J->C + bc_off(J->d, b, t, h, 0), N, nr ? nr->normw_C : NULL,
                   nr && nr->bias_C ? nr->bias_C + h * N : NULL, nr ? nr->eps : 0.0, tmp);
        rotate_pairs(tmp, phi, K, N, Cb);
        const double *xt = J->x + bth * P;
        for (long n = 0; n < N; n++)
            for (long p = 0; p < P; p++) {
                double u = Bb[n] * xt[p];
                hs[n * P + p] = al * hs[n * P + p] + be * Up[n * P + p] + ga * u;
                Up[n * P + p] = u;
            }
        double *yt = J->y + bth * P;
        for (long p = 0; p < P; p++) {
            double acc = 0.0;
            for (long n = 0; n < N; n++) acc += Cb[n] * hs[n * P + p];
            yt[p] = acc + J->D[h] * xt[p];
        }
    }
    if (J->h_out) memcpy(J->h_out + lane * NP, hs, sizeof(double) * NP);
    if (J->prevBx_out) memcpy(J->prevBx_out + lane * NP, Up, sizeof(double) * NP);
    if (J->angle_out) memcpy(J->angle_out + lane * K, phi, sizeof(double) * K);
    free(hs); free(Up); free(phi); free(tmp); free(Bb); free(Cb);
}

/* MIMO recurrence for one lane (torchmamba "Models": rank-R update on a
 * shared (N,P) state; "Math notes" App. C: per-head x/y expand by learned
 * vectors; dotLLM "MIMO streaming decode": state rank-summed, angle
 * rank-free):
 *   X_{t,r}[p] = W_x[h,r,p] x_t[p]
 *   U_t        = sum_r B_rot_{t,r} X_{t,r}^T
 *   h_t        = alpha_t h_{t-1} + beta_t U_{t-1} + gamma_t U_t
 *   y_t[p]     = sum_r W_y[h,r,p] (C_rot_{t,r}^T h_t)[p] + D_h x_t[p]
 * NULL W_x / W_y mean all ones. */
static void mimo_lane(const lane_job *J, long b, long h)
{
    long T = J->d.seqlen, H = J->d.nheads, P = J->d.headdim, N = J->d.dstate;
    long R = J->d.rank;
    long NP = N * P;
    double *hs = (double *)xmalloc(sizeof(double) * NP);
    double *Up = (double *)xmalloc(sizeof(double) * NP);
    double *Ut = (double *)xmalloc(sizeof(double) * NP);
    long K = n_pairs(J->d);
    double *phi = (double *)xmalloc(sizeof(double) * K);
    double *tmp = (double *)xmalloc(sizeof(double) * N);
    double *Bb = (double *)xmalloc(sizeof(double) * R * N);
    double *Cb = (double *)xmalloc(sizeof(double) * R * N);
    double *Xr = (double *)xmalloc(sizeof(double) * R * P);
    long lane = b * H + h;
    for (long k = 0; k < NP; k++) {
        hs[k] = J->h0 ? J->h0[lane * NP + k] : 0.0;
        Up[k] = J->prevBx0 ? J->prevBx0[lane * NP + k] : 0.0;
    }
    for (long i = 0; i < K; i++)
        phi[i] = J->angle0 ? J->angle0[lane * K + i] : 0.0;
    const m3o_bcnorm *nr = J->nrm;
    for (long t = 0; t < T; t++) {
        long bth = (b * T + t) * H + h;
        double dl = J->dt[bth], lm = J->lam[bth];
        double al = exp(dl * J->A[h]);
        double be = (1.0 - lm) * dl * al;
        double ga = lm * dl;
        for (long i = 0; i < K; i++) phi[i] += dl * J->theta[bth * K + i];
        const double *xt = J->x + bth * P;
        for (long r = 0; r < R; r++) {
            long off = bc_off(J->d, b, t, h, r);
            bc_prepare(J->B + off, N, nr ? nr->normw_B : NULL,
                       nr && nr->bias_B ? nr->bias_B + (h * R + r) * N : NULL, nr ? nr->eps : 0.0, tmp);
            rotate_pairs(tmp, phi, K, N, Bb + r * N);
            bc_prepare(J->C + off, N, nr ? nr->normw_C : NULL,
                       nr && nr->bias_C ? nr->bias_C + (h * R + r) * N : NULL, nr ? nr->eps : 0.0, tmp);
            rotate_pairs(tmp, phi, K, N, Cb + r * N);
            for (long p = 0; p < P; p++)
                Xr[r * P + p] = (J->Wx ? J->Wx[(h * R + r) * P + p] : 1.0) * xt[p];
        }
        for (long n = 0; n < N; n++)
            for (long p = 0; p < P; p++) {
                double u = 0.0;
                for (long r = 0; r < R; r++) u += Bb[r * N + n] * Xr[r * P + p];
                Ut[n * P + p] = u;
            }
        for (long k = 0; k < NP; k++) {
            hs[k] = al * hs[k] + be * Up[k] + ga * Ut[k];
            Up[k] = Ut[k];
        }
        double *yt = J->y + bth * P;
        for (long p = 0; p < P; p++) {
            double acc = 0.0;
            for (long r = 0; r < R; r++) {
                double yr = 0.0;
                for (long n = 0; n < N; n++) yr += Cb[r * N + n] * hs[n * P + p];
                acc += (J->Wy ? J->Wy[(h * R + r) * P + p] : 1.0) * yr;
            }
            yt[p] = acc + J->D[h] * xt[p];
        }
    }
    if (J->h_out) memcpy(J->h_out + lane * NP, hs, sizeof(double) * NP);
    if (J->prevBx_out) memcpy(J->prevBx_out + lane * NP, Up, sizeof(double) * NP);
    if (J->angle_out) memcpy(J->angle_out + lane * K, phi, sizeof(double) * K);
    free(hs); free(Up); free(Ut); free(phi); free(tmp); free(Bb); free(Cb); free(Xr);
}

/* Chunked form of the SISO scan, fp64, used only to self-test the
 * shifted-gamma fold (dotLLM streaming-decode comment: shifted_gamma[t] =
 * DT[t+1](1-trap[t+1]), scale = gamma + shifted_gamma, boundary fold
 * DT[0](1-trap[0]) before the scan's alpha; torchmamba "Math notes": Mamba-2
 * chunkwise intra-chunk quadratic part plus a factored inter-chunk carry).
 *   g_t = h_t + sg_t U_t  with  sg_t = (1-lam_{t+1}) dt_{t+1}  (0 at t=T-1)
 *   g_t = alpha_t g_{t-1} + w_t U_t,   w_t = gamma_t + sg_t
 *   g_{-1} = h0 + (1-lam_0) dt_0 prev_Bx0
 * Inside a chunk [t0, t1), with cum_t = sum_{k=t0..t} log alpha_k:
 *   y_t  = e^{cum_t} C_t^T g_in + sum_{s<=t} M[t,s] (C_t.B_s) x_s + D x_t
 *   M[t,s] = e^{cum_t - cum_s} w_s (s < t),  gamma_t (s == t)
 *   g_out = e^{cum_end} g_in + sum_s e^{cum_end - cum_s} w_s B_s x_s^T
 * At the end h_final = g_{T-1} and prev_Bx = B_{T-1} x_{T-1}^T. */
static void siso_chunked_lane(const lane_job *J, long b, long h)
{
    long T = J->d.seqlen, H = J->d.nheads, P = J->d.headdim, N = J->d.dstate;
    long Q = J->chunk;
    long NP = N * P;
    long lane = b * H + h;
    const m3o_bcnorm *nr = J->nrm;
    double *Bb = (double *)xmalloc(sizeof(double) * T * N);
    double *Cb = (double *)xmalloc(sizeof(double) * T * N);
    long K = n_pairs(J->d);
    double *phi = (double *)xmalloc(sizeof(double) * K);
    double *tmp = (double *)xmalloc(sizeof(double) * N);
    double *la = (double *)xmalloc(sizeof(double) * T);   /* log alpha */
    double *ga = (double *)xmalloc(sizeof(double) * T);
    double *w = (double *)xmalloc(sizeof(double) * T);
    double *g = (double *)xmalloc(sizeof(double) * NP);
    double *gn = (double *)xmalloc(sizeof(double) * NP);
    double *cum = (double *)xmalloc(sizeof(double) * Q);
    for (long i = 0; i < K; i++)
        phi[i] = J->angle0 ? J->angle0[lane * K + i] : 0.0;
    for (long t = 0; t < T; t++) {
        long bth = (b * T + t) * H + h;
        double dl = J->dt[bth];
        for (long i = 0; i < K; i++) phi[i] += dl * J->theta[bth * K + i];
        bc_prepare(J->B + bc_off(J->d, b, t, h, 0), N, nr ? nr->normw_B : NULL,
                   nr && nr->bias_B ? nr->bias_B + h * N : NULL, nr ? nr->eps : 0.0, tmp);
        rotate_pairs(tmp, phi, K, N, Bb + t * N);
        bc_prepare(J->C + bc_off(J->d, b, t, h, 0), N, nr ? nr->normw_C : NULL,
                   nr && nr->bias_C ? nr->bias_C + h * N : NULL, nr ? nr->eps : 0.0, tmp);
        rotate_pairs(tmp, phi, K, N, Cb + t * N);
        la[t] = dl * J->A[h];
        ga[t] = J->lam[bth] * dl;
    }
    for (long t = 0; t < T; t++) {
        double sg = 0.0;
        if (t + 1 < T) {
            long nx = (b * T + t + 1) * H + h;
            sg = (1.0 - J->lam[nx]) * J->dt[nx];
        }
        w[t] = ga[t] + sg;
    }
    {
        long b0 = (b * T + 0) * H + h;
        double f = T > 0 ? (1.0 - J->lam[b0]) * J->dt[b0] : 0.0;
        for (long k = 0; k < NP; k++)
            g[k] = (J->h0 ? J->h0[lane * NP + k] : 0.0) +
                   f * (J->prevBx0 ? J->prevBx0[lane * NP + k] : 0.0);
    }
    for (long t0 = 0; t0 < T; t0 += Q) {
        long t1 = t0 + Q < T ? t0 + Q : T;
        double run = 0.0;
        for (long t = t0; t < t1; t++) { run += la[t]; cum[t - t0] = run; }
        double cend = cum[t1 - 1 - t0];
        for (long t = t0; t < t1; t++) {
            long bth = (b * T + t) * H + h;
            double et = exp(cum[t - t0]);
            for (long p = 0; p < P; p++) {
                double acc = 0.0;
                for (long n = 0; n < N; n++) acc += Cb[t * N + n] * g[n * P + p];
                acc *= et;
                for (long s = t0; s <= t; s++) {
                    double cb = 0.0;
                    for (long n = 0; n < N; n++) cb += Cb[t * N + n] * Bb[s * N + n];
                    double m = (s == t) ? ga[t] : exp(cum[t - t0] - cum[s - t0]) * w[s];
                    acc += m * cb * J->x[((b * T + s) * H + h) * P + p];
                }
                J->y[bth * P + p] = acc + J->D[h] * J->x[bth * P + p];
            }
        }
        double ee = exp(cend);
        for (long n = 0; n < N; n++)
            for (long p = 0; p < P; p++) {
                double acc = ee * g[n * P + p];
                for (long s = t0; s < t1; s++)
                    acc += exp(cend - cum[s - t0]) * w[s] * Bb[s * N + n] *
                           J->x[((b * T + s) * H + h) * P + p];
                gn[n * P + p] = acc;
            }
        memcpy(g, gn, sizeof(double) * NP);
    }
    if (J->h_out) memcpy(J->h_out + lane * NP, g, sizeof(double) * NP);
    if (J->prevBx_out) {
        for (long n = 0; n < N; n++)
            for (long p = 0; p < P; p++)
                J->prevBx_out[lane * NP + n * P + p] =
                    T > 0 ? Bb[(T - 1) * N + n] * J->x[((b * T + T - 1) * H + h) * P + p]
                          : (J->prevBx0 ? J->prevBx0[lane * NP + n * P + p] : 0.0);
    }
    if (J->angle_out) memcpy(J->angle_out + lane * K, phi, sizeof(double) * K);
    free(Bb); free(Cb); free(phi); free(tmp); free(la); free(ga); free(w);
    free(g); free(gn); free(cum);
}

static void *lane_worker(void *arg)
{
    lane_job *J = (lane_job *)arg;
    long H = J->d.nheads;
    for (long lane = J->lane_begin; lane < J->lane_end; lane++) {
        long b = lane / H, h = lane % H;
        if (J->kind == 0) siso_lane(J, b, h);
        else if (J->kind == 1) mimo_lane(J, b, h);
        else siso_chunked_lane(J, b, h);
    }
    return NULL;
}

static int run_lanes(lane_job *proto, int nthreads)
{
    long lanes = proto->d.batch * proto->d.nheads;
    if (lanes <= 0) return 0;
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > lanes) nthreads = (int)lanes;
    pthread_t *th = (pthread_t *)xmalloc(sizeof(pthread_t) * nthreads);
    lane_job *jobs = (lane_job *)xmalloc(sizeof(lane_job) * nthreads);
    for (int i = 0; i < nthreads; i++) {
        jobs[i] = *proto;
        jobs[i].lane_begin = lanes * i / nthreads;
        jobs[i].lane_end = lanes * (i + 1) / nthreads;
    }
    char *started = (char *)xmalloc((size_t)nthreads);
    for (int i = 1; i < nthreads; i++) started[i] = pthread_create(&th[i], NULL, lane_worker, &jobs[i]) == 0;
    lane_worker(&jobs[0]);
    /* a job whose thread could not start runs here, so every lane is done */
    for (int i = 1; i < nthreads; i++) {
        if (started[i]) pthread_join(th[i], NULL);
        else lane_worker(&jobs[i]);
    }
    free(started);
    free(th);
    free(jobs);
    return nthreads;
}

static int check_dims(m3o_dims d, int mimo)
{
    if (d.batch < 0 || d.seqlen < 0 || d.nheads <= 0 || d.headdim <= 0) return -1;
    if (d.dstate <= 0 || (d.dstate & 1)) return -1;  /* RoPE needs even N */
    if (mimo && d.rank < 1) return -1;
    if (d.ngroups < 0 || d.rope_pairs < 0) return -1;
    if (d.nheads % n_groups(d)) return -1;              /* H % G == 0 */
    if (n_pairs(d) > d.dstate / 2) return -1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Public oracle entry points.  Each returns the number of threads used     */
/* (>= 1), 0 when there is no lane to run, or -1 on a bad argument.         */
/* ------------------------------------------------------------------------ */
int m3o_siso_loop(const double *x, const double *dt, const double *A,
                  const double *lam, const double *theta, const double *B,
                  const double *C, const double *D, const m3o_bcnorm *nrm,
                  const double *h0, const double *prevBx0, const double *angle0,
                  m3o_dims d, double *y, double *h_out, double *prevBx_out,
                  double *angle_out, int nthreads)
{
    if (check_dims(d, 0)) return -1;
    if (!x || !dt || !A || !lam || !theta || !B || !C || !D || !y) return -1;
    lane_job J;
    memset(&J, 0, sizeof J);
    J.x = x; J.dt = dt; J.A = A; J.lam = lam; J.theta = theta; J.B = B; J.C = C;
    J.D = D; J.nrm = nrm; J.h0 = h0; J.prevBx0 = prevBx0; J.angle0 = angle0;
    J.d = d; J.d.rank = 1; J.y = y; J.h_out = h_out; J.prevBx_out = prevBx_out;
    J.angle_out = angle_out; J.kind = 0;
    return run_lanes(&J, nthreads);
}

int m3o_mimo_loop(const double *x, const double *dt, const double *A,
                  const double *lam, const double *theta, const double *B,
                  const double *C, const double *D, const double *Wx,
                  const double *Wy, const m3o_bcnorm *nrm, const double *h0,
                  const double *prevBx0, const double *angle0, m3o_dims d,
                  double *y, double *h_out, double *prevBx_out,
                  double *angle_out, int nthreads)
{
    if (check_dims(d, 1)) return -1;
    if (!x || !dt || !A || !lam || !theta || !B || !C || !D || !y) return -1;
    lane_job J;
    memset(&J, 0, sizeof J);
    J.x = x; J.dt = dt; J.A = A; J.lam = lam; J.theta = theta; J.B = B; J.C = C;
    J.D = D; J.Wx = Wx; J.Wy = Wy; J.nrm = nrm; J.h0 = h0; J.prevBx0 = prevBx0;
    J.angle0 = angle0; J.d = d; J.y = y; J.h_out = h_out;
    J.prevBx_out = prevBx_out; J.angle_out = angle_out; J.kind = 1;
    return run_lanes(&J, nthreads);
}

int m3o_siso_chunked(const double *x, const double *dt, const double *A,
                     const double *lam, const double *theta, const double *B,
                     const double *C, const double *D, const m3o_bcnorm *nrm,
                     const double *h0, const double *prevBx0,
                     const double *angle0, m3o_dims d, long chunk, double *y,
                     double *h_out, double *prevBx_out, double *angle_out,
                     int nthreads)
{
    if (check_dims(d, 0) || chunk < 1) return -1;
    if (!x || !dt || !A || !lam || !theta || !B || !C || !D || !y) return -1;
    lane_job J;
    memset(&J, 0, sizeof J);
    J.x = x; J.dt = dt; J.A = A; J.lam = lam; J.theta = theta; J.B = B; J.C = C;
    J.D = D; J.nrm = nrm; J.h0 = h0; J.prevBx0 = prevBx0; J.angle0 = angle0;
    J.d = d; J.d.rank = 1; J.y = y; J.h_out = h_out; J.prevBx_out = prevBx_out;
    J.angle_out = angle_out; J.kind = 2; J.chunk = chunk;
    return run_lanes(&J, nthreads);
}

/* One decode step (SISO): the loop body for a single token, carrying
 * (h, prev_Bx, angle) in place.  Per-token inputs are shaped as a
 * one-token sequence: x (Bt,1,H,P), dt/lam (Bt,1,H), theta (Bt,1,H,K),
 * B/C (Bt,1,G,N); y (Bt,1,H,P). */
int m3o_step_decode(const double *x, const double *dt, const double *A,
                    const double *lam, const double *theta, const double *B,
                    const double *C, const double *D, const m3o_bcnorm *nrm,
                    m3o_dims d, double *h, double *prevBx, double *angle,
                    double *y, int nthreads)
{
    if (!h || !prevBx || !angle) return -1;
    d.seqlen = 1;
    long lanes = d.batch * d.nheads, NP = d.dstate * d.headdim;
    double *h1 = (double *)xmalloc(sizeof(double) * (lanes * NP + 1));
    double *u1 = (double *)xmalloc(sizeof(double) * (lanes * NP + 1));
    double *a1 = (double *)xmalloc(sizeof(double) * (lanes * n_pairs(d) + 1));
    int rc = m3o_siso_loop(x, dt, A, lam, theta, B, C, D, nrm, h, prevBx, angle,
                           d, y, h1, u1, a1, nthreads);
    if (rc >= 0) {
        memcpy(h, h1, sizeof(double) * lanes * NP);
        memcpy(prevBx, u1, sizeof(double) * lanes * NP);
        memcpy(angle, a1, sizeof(double) * lanes * n_pairs(d));
    }
    free(h1); free(u1); free(a1);
    return rc;
}

/* One MIMO decode step (rank R, W_x/W_y may be NULL for all ones): the MIMO
 * loop body for a single token, carrying (h, prev_Bx, angle) in place
 * (dotLLM "Mamba-3 MIMO streaming decode": the state is rank-summed and the
 * angle rank-free).  Per-token inputs are shaped as a one-token sequence. */
int m3o_mimo_step_decode(const double *x, const double *dt, const double *A,
                         const double *lam, const double *theta, const double *B,
                         const double *C, const double *D, const double *Wx,
                         const double *Wy, const m3o_bcnorm *nrm, m3o_dims d,
                         double *h, double *prevBx, double *angle, double *y, int nthreads)
{
    if (!h || !prevBx || !angle) return -1;
    d.seqlen = 1;
    long lanes = d.batch * d.nheads, NP = d.dstate * d.headdim;
    double *h1 = (double *)xmalloc(sizeof(double) * (lanes * NP + 1));
    double *u1 = (double *)xmalloc(sizeof(double) * (lanes * NP + 1));
    double *a1 = (double *)xmalloc(sizeof(double) * (lanes * n_pairs(d) + 1));
    int rc = m3o_mimo_loop(x, dt, A, lam, theta, B, C, D, Wx, Wy, nrm, h, prevBx, angle,
                           d, y, h1, u1, a1, nthreads);
    if (rc >= 0) {
        memcpy(h, h1, sizeof(double) * lanes * NP);
        memcpy(prevBx, u1, sizeof(double) * lanes * NP);
        memcpy(angle, a1, sizeof(double) * lanes * n_pairs(d));
    }
    free(h1); free(u1); free(a1);
    return rc;
}

/* One decode step on the factored previous-input state (torchmamba "Models":
 * the SISO cache carries (angle, ssm, x_prev, b_prev); dotLLM "Mamba-3 MIMO
 * streaming decode": per-rank key/value states instead of their product).
 * The previous token's input term is rebuilt from its factors,
 *   U_prev[n][p] = sum_r b_prev[r][n] W_x[h,r,p] x_prev[p],
 * the step is the MIMO recurrence for one token (rank 1 with W = 1 is the
 * SISO step), and afterwards b_prev <- B_rot_{t,r}, x_prev <- x_t.
 * In/out: h (Bt,H,N,P), bprev (Bt,H,R,N), xprev (Bt,H,P), angle (Bt,H,K).
 * Inputs: x (Bt,H,P), dt/lam (Bt,H), theta (Bt,H,K), B/C (Bt,G,R,N),
 * W_x/W_y (H,R,P) or NULL.  Output y (Bt,H,P). */
int m3o_step_decode_factored(const double *x, const double *dt, const double *A,
                             const double *lam, const double *theta, const double *B,
                             const double *C, const double *D, const double *Wx,
                             const double *Wy, const m3o_bcnorm *nrm, m3o_dims d,
                             double *h, double *bprev, double *xprev, double *angle,
                             double *y)
{
    if (!h || !bprev || !xprev || !angle || !x || !dt || !A || !lam || !theta || !B || !C || !D || !y)
        return -1;
    if (d.batch < 0 || d.nheads <= 0 || d.headdim <= 0 || d.dstate <= 0 || d.dstate % 2 || d.rank < 1)
        return -1;
    if (d.ngroups < 0 || d.rope_pairs < 0 || d.nheads % n_groups(d) || n_pairs(d) > d.dstate / 2)
        return -1;
    d.seqlen = 1;
    long H = d.nheads, P = d.headdim, N = d.dstate, R = d.rank, NP = N * P, K = n_pairs(d);
    double *tmp = (double *)xmalloc(sizeof(double) * N);
    double *Bb = (double *)xmalloc(sizeof(double) * R * N);
    double *Cb = (double *)xmalloc(sizeof(double) * R * N);
    double *Xr = (double *)xmalloc(sizeof(double) * R * P);
    double *Xp = (double *)xmalloc(sizeof(double) * R * P);
    for (long lane = 0; lane < d.batch * H; lane++) {
        long hh = lane % H;
        double dl = dt[lane], lm = lam[lane];
        double al = exp(dl * A[hh]);
        double be = (1.0 - lm) * dl * al;
        double ga = lm * dl;
        double *phi = angle + lane * K;
        for (long i = 0; i < K; i++) phi[i] += dl * theta[lane * K + i];
        const double *xt = x + lane * P;
        double *xo = xprev + lane * P;
        for (long r = 0; r < R; r++) {
            long off = bc_off(d, lane / H, 0, hh, r);
            bc_prepare(B + off, N, nrm ? nrm->normw_B : NULL,
                       nrm && nrm->bias_B ? nrm->bias_B + (hh * R + r) * N : NULL, nrm ? nrm->eps : 0.0, tmp);
            rotate_pairs(tmp, phi, K, N, Bb + r * N);
            bc_prepare(C + off, N, nrm ? nrm->normw_C : NULL,
                       nrm && nrm->bias_C ? nrm->bias_C + (hh * R + r) * N : NULL, nrm ? nrm->eps : 0.0, tmp);
            rotate_pairs(tmp, phi, K, N, Cb + r * N);
            for (long p = 0; p < P; p++) {
                double w = Wx ? Wx[(hh * R + r) * P + p] : 1.0;
                Xr[r * P + p] = w * xt[p];
                Xp[r * P + p] = w * xo[p];
            }
        }
        double *hs = h + lane * NP;
        const double *bp = bprev + lane * R * N;
        for (long n = 0; n < N; n++)
            for (long p = 0; p < P; p++) {
                double up = 0.0, ut = 0.0;
                for (long r = 0; r < R; r++) {
                    up += bp[r * N + n] * Xp[r * P + p];
                    ut += Bb[r * N + n] * Xr[r * P + p];
                }
                hs[n * P + p] = al * hs[n * P + p] + be * up + ga * ut;
            }
        double *yt = y + lane * P;
        for (long p = 0; p < P; p++) {
            double acc = 0.0;
            for (long r = 0; r < R; r++) {
                double yr = 0.0;
                for (long n = 0; n < N; n++) yr += Cb[r * N + n] * hs[n * P + p];
                acc += (Wy ? Wy[(hh * R + r) * P + p] : 1.0) * yr;
            }
            yt[p] = acc + D[hh] * xt[p];
        }
        memcpy(bprev + lane * R * N, Bb, sizeof(double) * R * N);
        memcpy(xo, xt, sizeof(double) * P);
    }
    free(tmp); free(Bb); free(Cb); free(Xr); free(Xp);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Backward: the gradient of the scan's outputs with respect to every input */
/* (training needs it: TorchMamba README, "Models" and "Verification";      */
/* dotLLM pull request, the note that training is out of its scope).         */
/*                                                                            */
/* The loss is L = <dy, y> + <dh_final, h_{T-1}> + <dprevBx, U_{T-1}> +      */
/* <dangle, Phi_{T-1}> (each seed may be NULL for zero).  This is the       */
/* reverse sweep of the rank-R loop above, one lane at a time, with the     */
/* forward values of the lane kept in memory:                                */
/*   Gh_t  = adjoint of h_t = alpha_{t+1} Gh_{t+1} + sum_r C_rot_{t,r}        */
/*           (W_y[r] dy_t)^T       (Gh_{T-1} starts from dh_final)          */
/*   GU_t  = adjoint of U_t = gamma_t Gh_t + beta_{t+1} Gh_{t+1}             */
/*           (dprevBx at t = T-1)                                            */
/*   dalpha_t = <Gh_t, h_{t-1}>, dbeta_t = <Gh_t, U_{t-1}>,                 */
/*   dgamma_t = <Gh_t, U_t>;  dh0 = alpha_0 Gh_0, dprevBx0 = beta_0 Gh_0;    */
/*   a rotation by Phi turns the pair adjoint back by -Phi and adds          */
/*   -dv[2i] v_rot[2i+1] + dv[2i+1] v_rot[2i] to the adjoint of Phi_t[i],     */
/*   which flows unchanged to Phi_{t-1} and gives dtheta_t = dt_t GPhi_t,    */
/*   ddt_t += <theta_t, GPhi_t>;  dangle0 = GPhi_0.                          */
/* Every gradient buffer may be NULL (not wanted); the others are            */
/* overwritten.  Shared parameters (A, D, W_x, W_y, the norm gains and       */
/* biases, and grouped B/C rows) sum over the lanes that use them.           */
/* ------------------------------------------------------------------------ */
typedef struct {
    double *dx, *ddt, *dA, *dlam, *dtheta, *dB, *dC, *dD, *dWx, *dWy;
    double *dnormw_B, *dnormw_C, *dbias_B, *dbias_C;
    double *dh0, *dprevBx0, *dangle0;
} m3o_grads;

static void zero_if(double *p, long n)
{
    if (p) memset(p, 0, sizeof(double) * (size_t)n);
}

/* adjoint of bc_prepare: dst = src * inv * w + bias (inv, w only with w) */
static void bc_prepare_bwd(const double *src, long N, const double *w, double eps,
                           const double *ddst, double *dsrc, double *dw, double *dbias)
{
    if (dbias)
        for (long n = 0; n < N; n++) dbias[n] += ddst[n];
    if (!w) {
        for (long n = 0; n < N; n++) dsrc[n] += ddst[n];
        return;
    }
    double ss = 0.0;
    for (long n = 0; n < N; n++) ss += src[n] * src[n];
    double inv = 1.0 / sqrt(ss / (double)N + eps);
    double s = 0.0;  /* sum_n ddst[n] w[n] src[n] */
    for (long n = 0; n < N; n++) {
        s += ddst[n] * w[n] * src[n];
        if (dw) dw[n] += ddst[n] * src[n] * inv;
    }
    for (long n = 0; n < N; n++)
        dsrc[n] += inv * ddst[n] * w[n] - src[n] * inv * inv * inv * s / (double)N;
}

int m3o_mimo_loop_bwd(const double *x, const double *dt, const double *A,
                      const double *lam, const double *theta, const double *B,
                      const double *C, const double *D, const double *Wx,
                      const double *Wy, const m3o_bcnorm *nrm, const double *h0,
                      const double *prevBx0, const double *angle0, m3o_dims d,
                      const double *dy, const double *dh_final,
                      const double *dprevBx_final, const double *dangle_final,
                      m3o_grads *g)
{
    if (check_dims(d, 1)) return -1;
    if (!x || !dt || !A || !lam || !theta || !B || !C || !D || !g) return -1;
    long Bt = d.batch, T = d.seqlen, H = d.nheads, P = d.headdim, N = d.dstate, R = d.rank;
    long K = n_pairs(d), G = n_groups(d), NP = N * P;
    long RN = R * N, RP = R * P;
    zero_if(g->dx, Bt * T * H * P);
    zero_if(g->ddt, Bt * T * H);
    zero_if(g->dA, H);
    zero_if(g->dlam, Bt * T * H);
    zero_if(g->dtheta, Bt * T * H * K);
    zero_if(g->dB, Bt * T * G * RN);
    zero_if(g->dC, Bt * T * G * RN);
    zero_if(g->dD, H);
    zero_if(g->dWx, H * RP);
    zero_if(g->dWy, H * RP);
    zero_if(g->dnormw_B, N);
    zero_if(g->dnormw_C, N);
    zero_if(g->dbias_B, H * RN);
    zero_if(g->dbias_C, H * RN);
    zero_if(g->dh0, Bt * H * NP);
    zero_if(g->dprevBx0, Bt * H * NP);
    zero_if(g->dangle0, Bt * H * K);
    double eps = nrm ? nrm->eps : 0.0;
    const double *wB = nrm ? nrm->normw_B : NULL, *wC = nrm ? nrm->normw_C : NULL;

    double *phis = (double *)xmalloc(sizeof(double) * (T + 1) * K);   /* Phi_{t-1}, t = 0..T */
    double *Bp = (double *)xmalloc(sizeof(double) * (T * RN + 1));    /* QkNorm'd + bias'd */
    double *Cp = (double *)xmalloc(sizeof(double) * (T * RN + 1));
    double *Bb = (double *)xmalloc(sizeof(double) * (T * RN + 1));    /* rotated */
    double *Cb = (double *)xmalloc(sizeof(double) * (T * RN + 1));
    double *X = (double *)xmalloc(sizeof(double) * (T * RP + 1));     /* W_x[r] x_t */
    double *al = (double *)xmalloc(sizeof(double) * (T + 1));
    double *be = (double *)xmalloc(sizeof(double) * (T + 1));
    double *ga = (double *)xmalloc(sizeof(double) * (T + 1));
    double *hs = (double *)xmalloc(sizeof(double) * (T + 1) * NP);    /* h_{t-1}, t = 0..T */
    double *Ut = (double *)xmalloc(sizeof(double) * NP);
    double *Um = (double *)xmalloc(sizeof(double) * NP);
    double *Gh = (double *)xmalloc(sizeof(double) * NP);
    double *GU = (double *)xmalloc(sizeof(double) * NP);
    double *GUf = (double *)xmalloc(sizeof(double) * NP);
    double *Gphi = (double *)xmalloc(sizeof(double) * K);
    double *dBb = (double *)xmalloc(sizeof(double) * RN);
    double *dCb = (double *)xmalloc(sizeof(double) * RN);
    double *dBp = (double *)xmalloc(sizeof(double) * N);
    double *dCp = (double *)xmalloc(sizeof(double) * N);
    double *dX = (double *)xmalloc(sizeof(double) * RP);
    double *tmp = (double *)xmalloc(sizeof(double) * N);

    for (long b = 0; b < Bt; b++)
        for (long h = 0; h < H; h++) {
            long lane = b * H + h;
            /* ---- forward, keeping what the reverse sweep needs ---- */
            for (long i = 0; i < K; i++) phis[i] = angle0 ? angle0[lane * K + i] : 0.0;
            for (long k = 0; k < NP; k++) hs[k] = h0 ? h0[lane * NP + k] : 0.0;
            for (long k = 0; k < NP; k++) Um[k] = prevBx0 ? prevBx0[lane * NP + k] : 0.0;
            for (long t = 0; t < T; t++) {
                long bth = (b * T + t) * H + h;
                double dl = dt[bth], lm = lam[bth];
                al[t] = exp(dl * A[h]);
                be[t] = (1.0 - lm) * dl * al[t];
                ga[t] = lm * dl;
                double *phi = phis + (t + 1) * K;
                for (long i = 0; i < K; i++) phi[i] = phis[t * K + i] + dl * theta[bth * K + i];
                for (long r = 0; r < R; r++) {
                    long off = bc_off(d, b, t, h, r);
                    bc_prepare(B + off, N, wB, nrm && nrm->bias_B ? nrm->bias_B + (h * R + r) * N : NULL, eps,
                               Bp + (t * R + r) * N);
                    bc_prepare(C + off, N, wC, nrm && nrm->bias_C ? nrm->bias_C + (h * R + r) * N : NULL, eps,
                               Cp + (t * R + r) * N);
                    rotate_pairs(Bp + (t * R + r) * N, phi, K, N, Bb + (t * R + r) * N);
                    rotate_pairs(Cp + (t * R + r) * N, phi, K, N, Cb + (t * R + r) * N);
                    for (long p = 0; p < P; p++)
                        X[(t * R + r) * P + p] = (Wx ? Wx[(h * R + r) * P + p] : 1.0) * x[bth * P + p];
                }
                for (long n = 0; n < N; n++)
                    for (long p = 0; p < P; p++) {
                        double u = 0.0;
                        for (long r = 0; r < R; r++) u += Bb[(t * R + r) * N + n] * X[(t * R + r) * P + p];
                        hs[(t + 1) * NP + n * P + p] = al[t] * hs[t * NP + n * P + p] + be[t] * Um[n * P + p] +
                                                       ga[t] * u;
                        Ut[n * P + p] = u;
                    }
                memcpy(Um, Ut, sizeof(double) * NP);
            }
            /* ---- reverse sweep ---- */
            for (long k = 0; k < NP; k++) {
                Gh[k] = dh_final ? dh_final[lane * NP + k] : 0.0;
                GUf[k] = dprevBx_final ? dprevBx_final[lane * NP + k] : 0.0;
            }
            for (long i = 0; i < K; i++) Gphi[i] = dangle_final ? dangle_final[lane * K + i] : 0.0;
            for (long t = T - 1; t >= 0; t--) {
                long bth = (b * T + t) * H + h;
                double dl = dt[bth], lm = lam[bth];
                const double *ht = hs + (t + 1) * NP, *hm = hs + t * NP;
                const double *dyt = dy ? dy + bth * P : NULL;
                const double *xt = x + bth * P;
                /* y_t = sum_r W_y[r] (C_rot_{t,r}^T h_t) + D x_t */
                for (long r = 0; r < R; r++)
                    for (long n = 0; n < N; n++) dCb[r * N + n] = 0.0;
                if (dyt) {
                    for (long r = 0; r < R; r++) {
                        const double *cb = Cb + (t * R + r) * N;
                        for (long p = 0; p < P; p++) {
                            double wy = Wy ? Wy[(h * R + r) * P + p] : 1.0;
                            double yr = 0.0;
                            for (long n = 0; n < N; n++) {
                                yr += cb[n] * ht[n * P + p];
                                Gh[n * P + p] += cb[n] * wy * dyt[p];
                                dCb[r * N + n] += wy * dyt[p] * ht[n * P + p];
                            }
                            if (g->dWy) g->dWy[(h * R + r) * P + p] += dyt[p] * yr;
                        }
                    }
                    for (long p = 0; p < P; p++) {
                        if (g->dD) g->dD[h] += dyt[p] * xt[p];
                        if (g->dx) g->dx[bth * P + p] += D[h] * dyt[p];
                    }
                }
                /* h_t = alpha h_{t-1} + beta U_{t-1} + gamma U_t */
                double dal = 0.0, dbe = 0.0, dga = 0.0;
                for (long n = 0; n < N; n++)
                    for (long p = 0; p < P; p++) {
                        double u = 0.0, um = 0.0;
                        for (long r = 0; r < R; r++) {
                            u += Bb[(t * R + r) * N + n] * X[(t * R + r) * P + p];
                            if (t > 0) um += Bb[((t - 1) * R + r) * N + n] * X[((t - 1) * R + r) * P + p];
                        }
                        if (t == 0) um = prevBx0 ? prevBx0[lane * NP + n * P + p] : 0.0;
                        double gh = Gh[n * P + p];
                        dal += gh * hm[n * P + p];
                        dbe += gh * um;
                        dga += gh * u;
                        GU[n * P + p] = ga[t] * gh + GUf[n * P + p];
                    }
                /* U_t = sum_r B_rot_{t,r} X_{t,r}^T */
                for (long r = 0; r < R; r++) {
                    const double *bb = Bb + (t * R + r) * N, *xr = X + (t * R + r) * P;
                    for (long n = 0; n < N; n++) {
                        double s = 0.0;
                        for (long p = 0; p < P; p++) s += GU[n * P + p] * xr[p];
                        dBb[r * N + n] = s;
                    }
                    for (long p = 0; p < P; p++) {
                        double s = 0.0;
                        for (long n = 0; n < N; n++) s += GU[n * P + p] * bb[n];
                        dX[r * P + p] = s;
                        double wx = Wx ? Wx[(h * R + r) * P + p] : 1.0;
                        if (g->dx) g->dx[bth * P + p] += wx * s;
                        if (g->dWx) g->dWx[(h * R + r) * P + p] += xt[p] * s;
                    }
                }
                /* hand the state adjoints to step t-1 */
                for (long k = 0; k < NP; k++) {
                    GUf[k] = be[t] * Gh[k];
                    Gh[k] = al[t] * Gh[k];
                }
                /* discretization: alpha = e^{dt A}, beta = (1-lam) dt alpha, gamma = lam dt */
                double a = al[t];
                if (g->ddt) g->ddt[bth] += dal * A[h] * a + dbe * (1.0 - lm) * (a + dl * A[h] * a) + dga * lm;
                if (g->dA) g->dA[h] += dal * dl * a + dbe * (1.0 - lm) * dl * dl * a;
                if (g->dlam) g->dlam[bth] += -dbe * dl * a + dga * dl;
                /* rotation by Phi_t: angle adjoint and the un-rotated pair adjoints */
                const double *phi = phis + (t + 1) * K;
                for (long i = 0; i < K; i++) {
                    double gp = 0.0;
                    for (long r = 0; r < R; r++) {
                        const double *bb = Bb + (t * R + r) * N, *cb = Cb + (t * R + r) * N;
                        const double *db = dBb + r * N, *dc = dCb + r * N;
                        gp += -db[2 * i] * bb[2 * i + 1] + db[2 * i + 1] * bb[2 * i];
                        gp += -dc[2 * i] * cb[2 * i + 1] + dc[2 * i + 1] * cb[2 * i];
                    }
                    Gphi[i] += gp;
                    if (g->dtheta) g->dtheta[bth * K + i] += dl * Gphi[i];
                    if (g->ddt) g->ddt[bth] += theta[bth * K + i] * Gphi[i];
                }
                for (long r = 0; r < R; r++) {
                    const double *db = dBb + r * N, *dc = dCb + r * N;
                    for (long i = 0; i < K; i++) {
                        double c = cos(phi[i]), s = sin(phi[i]);
                        dBp[2 * i] = c * db[2 * i] + s * db[2 * i + 1];
                        dBp[2 * i + 1] = -s * db[2 * i] + c * db[2 * i + 1];
                        dCp[2 * i] = c * dc[2 * i] + s * dc[2 * i + 1];
                        dCp[2 * i + 1] = -s * dc[2 * i] + c * dc[2 * i + 1];
                    }
                    for (long n = 2 * K; n < N; n++) {
                        dBp[n] = db[n];
                        dCp[n] = dc[n];
                    }
                    long off = bc_off(d, b, t, h, r);
                    for (long n = 0; n < N; n++) tmp[n] = 0.0;
                    bc_prepare_bwd(B + off, N, wB, eps, dBp, tmp, g->dnormw_B,
                                   g->dbias_B && nrm && nrm->bias_B ? g->dbias_B + (h * R + r) * N : NULL);
                    if (g->dB)
                        for (long n = 0; n < N; n++) g->dB[off + n] += tmp[n];
                    for (long n = 0; n < N; n++) tmp[n] = 0.0;
                    bc_prepare_bwd(C + off, N, wC, eps, dCp, tmp, g->dnormw_C,
                                   g->dbias_C && nrm && nrm->bias_C ? g->dbias_C + (h * R + r) * N : NULL);
                    if (g->dC)
                        for (long n = 0; n < N; n++) g->dC[off + n] += tmp[n];
                }
            }
            /* the adjoints of the initial state: h_{-1} = h0, U_{-1} = prev_Bx0 */
            if (g->dh0) memcpy(g->dh0 + lane * NP, Gh, sizeof(double) * NP);
            if (g->dprevBx0) memcpy(g->dprevBx0 + lane * NP, GUf, sizeof(double) * NP);
            if (g->dangle0) memcpy(g->dangle0 + lane * K, Gphi, sizeof(double) * K);
        }
    free(phis); free(Bp); free(Cp); free(Bb); free(Cb); free(X); free(al); free(be); free(ga);
    free(hs); free(Ut); free(Um); free(Gh); free(GU); free(GUf); free(Gphi); free(dBb); free(dCb);
    free(dBp); free(dCp); free(dX); free(tmp);
    return 0;
}
