// m3_api.cu -- the C ABI declared in include/m3.h: argument validation on
// the host, then kernel launches on the caller's stream.  Nothing here
// allocates, frees or synchronises.
#include <atomic>
#include <cmath>
#include <initializer_list>

#include "m3_internal.cuh"

namespace m3 {
static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace m3

using namespace m3;

namespace {

constexpr int64_t kMaxDstate = 256, kMaxHeaddim = 256, kMaxStateElems = 16384, kMaxRank = 8;
// Every kernel runs one CTA per (batch, head) lane in a 1-D grid, and no
// tensor may hold more than 2^46 elements (far beyond device memory), so
// that every index product below stays well inside int64.
constexpr int64_t kMaxLanes = 0x7fffffff, kMaxElems = (int64_t)1 << 46;

// Product of non-negative sizes, saturated at kMaxElems + 1.
int64_t sat_product(std::initializer_list<int64_t> f) {
    for (int64_t v : f)
        if (v == 0) return 0;
    int64_t p = 1;
    for (int64_t v : f) {
        if (v > kMaxElems || p > kMaxElems / v) return kMaxElems + 1;
        p *= v;
    }
    return p;
}

// The requested chunk as an int: any request of 2^30 tokens or more behaves
// as 2^30 (longer than any supported sequence).
inline int chunk_request(int64_t c) { return (int)(c < ((int64_t)1 << 30) ? c : ((int64_t)1 << 30)); }

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// required pointer: non-null and 16-byte aligned
#define M3_REQ(p)                                                  \
    do {                                                           \
        if (!(p) || !aligned16(p)) return M3_ERR_INVALID_ARG;      \
    } while (0)
// optional pointer: null, or 16-byte aligned
#define M3_OPT(p)                                                  \
    do {                                                           \
        if ((p) && !aligned16(p)) return M3_ERR_INVALID_ARG;       \
    } while (0)

m3_status check_dtype(m3_dtype t) {
    return (t == M3_F32 || t == M3_BF16) ? M3_OK : M3_ERR_INVALID_ARG;
}

// Sizes shared by the scan, rope and decode entry points.
m3_status check_core_dims(const m3_dims &d, bool need_seq) {
    if (d.batch < 0 || d.nheads < 1 || d.headdim < 1 || d.dstate < 2) return M3_ERR_INVALID_ARG;
    if (need_seq && d.seqlen < 0) return M3_ERR_INVALID_ARG;
    if (d.dstate & 1) return M3_ERR_INVALID_ARG;  // RoPE pairs need an even dstate
    if (d.dstate > kMaxDstate || d.headdim > kMaxHeaddim || d.dstate * d.headdim > kMaxStateElems)
        return M3_ERR_UNSUPPORTED;
    if (d.batch > (int64_t)1 << 24 || d.nheads > 4096 || (need_seq && d.seqlen > ((int64_t)1 << 31)))
        return M3_ERR_UNSUPPORTED;
    if (d.batch * d.nheads > kMaxLanes) return M3_ERR_UNSUPPORTED;
    const int64_t width = d.headdim > d.dstate ? d.headdim : d.dstate;
    if (need_seq && sat_product({d.batch, d.seqlen, d.nheads, width}) > kMaxElems) return M3_ERR_UNSUPPORTED;
    return M3_OK;
}

// B/C groups and rotated pairs, with 0 meaning one group per head and every
// pair (TorchMamba README, "Models": n_groups with H % G == 0; dotLLM pull
// request, real-checkpoint run: num_rope_angles of dstate).
m3_status resolve_groups(const m3_dims &d, int64_t &G, int64_t &K) {
    if (d.ngroups < 0 || d.rope_pairs < 0) return M3_ERR_INVALID_ARG;
    G = d.ngroups ? d.ngroups : d.nheads;
    K = d.rope_pairs ? d.rope_pairs : d.dstate / 2;
    if (d.nheads % G || K > d.dstate / 2) return M3_ERR_INVALID_ARG;
    return M3_OK;
}

m3_status read_norm(const m3_bcnorm *n, NormArgs &o) {
    o = NormArgs{nullptr, nullptr, nullptr, nullptr, 0.f};
    if (!n) return M3_OK;
    M3_OPT(n->normw_B);
    M3_OPT(n->normw_C);
    M3_OPT(n->bias_B);
    M3_OPT(n->bias_C);
    if ((n->normw_B || n->normw_C) && !(n->eps >= 0.f && std::isfinite(n->eps))) return M3_ERR_INVALID_ARG;
    o = NormArgs{n->normw_B, n->normw_C, n->bias_B, n->bias_C, n->eps};
    return M3_OK;
}

inline m3_status launched(cudaError_t e) { return e == cudaSuccess ? M3_OK : M3_ERR_CUDA; }

// Failure-injection hook (m3_debug_fail_next_launches): the next n calls that
// pass validation report a launch failure without launching anything.
std::atomic<int> g_fail_launches{0};
inline bool injected_failure() {
    int n = g_fail_launches.load(std::memory_order_relaxed);
    while (n > 0)
        if (g_fail_launches.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) return true;
    return false;
}

// Every entry point ends here, after its validation: the launch, or the
// injected failure in its place.
template <typename F>
inline m3_status launch_unless_injected(F &&launch) {
    if (injected_failure()) return M3_ERR_CUDA;
    return launched(launch());
}

m3_status chunked_common(const void *x, const float *dt, const float *A, const float *lam,
                         const float *theta, const void *B, const void *C, const float *D,
                         const float *Wx, const float *Wy, m3_dtype dtype, const m3_bcnorm *norm,
                         const float *h0, const float *prevBx0, const float *angle0, m3_dims d,
                         void *y, float *h_final, float *prevBx_final, float *angle_final,
                         void *workspace, size_t ws_bytes, void *stream, bool mimo) {
    m3_status st;
    if ((st = check_dtype(dtype)) != M3_OK) return st;
    if ((st = check_core_dims(d, true)) != M3_OK) return st;
    if (d.chunk < 1) return M3_ERR_INVALID_ARG;
    int64_t G, K;
    if ((st = resolve_groups(d, G, K)) != M3_OK) return st;
    const int64_t R = mimo ? d.rank : 1;
    if (mimo && d.rank < 1) return M3_ERR_INVALID_ARG;
    if (R > kMaxRank) return M3_ERR_UNSUPPORTED;
    M3_REQ(A);
    M3_REQ(D);
    const bool have_tokens = d.batch > 0 && d.seqlen > 0;
    if (have_tokens) {
        M3_REQ(x); M3_REQ(dt); M3_REQ(lam); M3_REQ(theta); M3_REQ(B); M3_REQ(C); M3_REQ(y);
    } else {
        M3_OPT(x); M3_OPT(dt); M3_OPT(lam); M3_OPT(theta); M3_OPT(B); M3_OPT(C); M3_OPT(y);
    }
    M3_OPT(Wx); M3_OPT(Wy); M3_OPT(h0); M3_OPT(prevBx0); M3_OPT(angle0);
    M3_OPT(h_final); M3_OPT(prevBx_final); M3_OPT(angle_final); M3_OPT(workspace);
    NormArgs nrm;
    if ((st = read_norm(norm, nrm)) != M3_OK) return st;
    const size_t need = m3_workspace_bytes(mimo ? M3_WS_MIMO : M3_WS_SISO, d, dtype);
    if (need > 0 && (!workspace || ws_bytes < need)) return M3_ERR_WORKSPACE;
    const int q = scan_simt_chunk(d.headdim, d.dstate, R, d.chunk);
    if (q < 1) return M3_ERR_UNSUPPORTED;
    if (d.batch == 0) return M3_OK;
    if (d.seqlen > ((int64_t)1 << 30)) return M3_ERR_UNSUPPORTED;

    ScanArgs a;
    a.x = x; a.B = B; a.C = C;
    a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.D = D; a.Wx = Wx; a.Wy = Wy;
    a.h0 = h0; a.prevBx0 = prevBx0; a.angle0 = angle0;
    a.nrm = nrm;
    a.y = y; a.h_out = h_final; a.prevBx_out = prevBx_final; a.angle_out = angle_final;
    a.Bt = d.batch; a.T = d.seqlen; a.H = d.nheads; a.P = d.headdim; a.N = d.dstate; a.R = R;
    a.G = G; a.K = K;
    a.mimo_layout = mimo ? 1 : 0;
    a.ws = workspace;
    a.Q = chunk_request(d.chunk);
    if (scan_tc_supported(a, dtype))
        return launch_unless_injected([&] { return launch_scan_tc(a, (cudaStream_t)stream); });
    a.Q = q;
    return launch_unless_injected([&] { return launch_scan_simt(a, dtype, (cudaStream_t)stream); });
}

}  // namespace

extern "C" {

m3_limits m3_get_limits(void) { return m3_limits{kMaxDstate, kMaxHeaddim, kMaxStateElems, kMaxRank}; }

uint64_t m3_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *m3_status_string(m3_status s) {
    switch (s) {
        case M3_OK: return "M3_OK: success";
        case M3_ERR_INVALID_ARG: return "M3_ERR_INVALID_ARG: null, misaligned or inconsistent argument";
        case M3_ERR_UNSUPPORTED: return "M3_ERR_UNSUPPORTED: sizes outside this build's limits";
        case M3_ERR_WORKSPACE: return "M3_ERR_WORKSPACE: workspace missing or too small";
        case M3_ERR_CUDA: return "M3_ERR_CUDA: a kernel launch failed";
        case M3_ERR_TIMEOUT: return "M3_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    }
    return "unknown m3_status";
}

m3_status m3_device_error(void *stream, int *site) {
    const int e = scan_tc_error_and_clear((cudaStream_t)stream);
    if (site) *site = e > 0 ? e : 0;
    if (e < 0) return M3_ERR_CUDA;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return M3_ERR_CUDA;
    return e ? M3_ERR_TIMEOUT : M3_OK;
}

void m3_debug_fail_next_launches(int n) { g_fail_launches.store(n > 0 ? n : 0, std::memory_order_relaxed); }

m3_status m3_selftest_bounded_wait(void *stream) {
    return launch_unless_injected(
        [&] { return launch_wait_selftest(M3_SELFTEST_SITE, (cudaStream_t)stream); });
}

size_t m3_workspace_bytes(int which, m3_dims d, m3_dtype dtype) {
    if (which == M3_WS_BWD_SISO || which == M3_WS_BWD_MIMO) {
        BwdArgs b{};
        if (check_core_dims(d, true) != M3_OK || d.chunk < 1 || resolve_groups(d, b.G, b.K) != M3_OK) return 0;
        b.Bt = d.batch; b.T = d.seqlen; b.H = d.nheads; b.P = d.headdim; b.N = d.dstate;
        b.R = which == M3_WS_BWD_MIMO ? (d.rank > 1 ? d.rank : 1) : 1;
        b.Q = (int)(d.chunk < 64 ? d.chunk : 64);
        return scan_bwd_workspace_bytes(b);
    }
    // only the tensor-core path uses scratch (long sequences over few lanes)
    if ((which != M3_WS_SISO && which != M3_WS_MIMO) || check_core_dims(d, true) != M3_OK || d.chunk < 1) return 0;
    ScanArgs a{};
    if (resolve_groups(d, a.G, a.K) != M3_OK) return 0;
    a.Bt = d.batch; a.T = d.seqlen; a.H = d.nheads; a.P = d.headdim; a.N = d.dstate;
    a.R = which == M3_WS_MIMO ? d.rank : 1;
    a.Q = chunk_request(d.chunk); a.mimo_layout = which == M3_WS_MIMO ? 1 : 0;
    if (!scan_tc_supported(a, dtype)) return 0;
    return scan_tc_workspace_bytes(d.batch, d.nheads, d.seqlen);
}

m3_status m3_discretize(const float *dt, const float *A, const float *lam, m3_dims d, float *alpha,
                        float *beta, float *gamma, void *stream) {
    if (d.batch < 0 || d.seqlen < 0 || d.nheads < 1) return M3_ERR_INVALID_ARG;
    if (sat_product({d.batch, d.seqlen, d.nheads}) > kMaxElems) return M3_ERR_UNSUPPORTED;
    M3_REQ(A);
    if (d.batch * d.seqlen == 0) return M3_OK;
    M3_REQ(dt); M3_REQ(lam); M3_REQ(alpha); M3_REQ(beta); M3_REQ(gamma);
    return launch_unless_injected([&] {
        return launch_discretize(dt, A, lam, d.batch, d.seqlen, d.nheads, alpha, beta, gamma, (cudaStream_t)stream);
    });
}

m3_status m3_rope_bc(const void *B, const void *C, m3_dtype dtype, const float *theta, const float *dt,
                     const float *angle0, const m3_bcnorm *norm, m3_dims d, void *B_rot, void *C_rot,
                     float *angle_final, void *stream) {
    m3_status st;
    if ((st = check_dtype(dtype)) != M3_OK) return st;
    if ((st = check_core_dims(d, true)) != M3_OK) return st;
    int64_t G, K;
    if ((st = resolve_groups(d, G, K)) != M3_OK) return st;
    const int64_t R = d.rank > 1 ? d.rank : 1;
    if (d.rank < 0) return M3_ERR_INVALID_ARG;
    if (R > kMaxRank) return M3_ERR_UNSUPPORTED;
    if (d.batch > 0 && d.seqlen > 0) {
        M3_REQ(B); M3_REQ(C); M3_REQ(theta); M3_REQ(dt); M3_REQ(B_rot); M3_REQ(C_rot);
    }
    M3_OPT(angle0); M3_OPT(angle_final);
    NormArgs nrm;
    if ((st = read_norm(norm, nrm)) != M3_OK) return st;
    if (d.batch == 0) return M3_OK;
    RopeArgs a;
    a.B = B; a.C = C; a.theta = theta; a.dt = dt; a.angle0 = angle0; a.nrm = nrm;
    a.Bo = B_rot; a.Co = C_rot; a.angle_out = angle_final;
    a.Bt = d.batch; a.T = d.seqlen; a.H = d.nheads; a.R = R; a.N = d.dstate; a.G = G; a.K = K;
    return launch_unless_injected([&] { return launch_rope(a, dtype, (cudaStream_t)stream); });
}

m3_status m3_siso_chunked_fwd(const void *x, const float *dt, const float *A, const float *lam,
                              const float *theta, const void *B, const void *C, const float *D,
                              m3_dtype dtype, const m3_bcnorm *norm, const float *h0,
                              const float *prevBx0, const float *angle0, m3_dims d, void *y,
                              float *h_final, float *prevBx_final, float *angle_final, void *workspace,
                              size_t workspace_bytes, void *stream) {
    return chunked_common(x, dt, A, lam, theta, B, C, D, nullptr, nullptr, dtype, norm, h0, prevBx0,
                          angle0, d, y, h_final, prevBx_final, angle_final, workspace, workspace_bytes,
                          stream, false);
}

m3_status m3_mimo_chunked_fwd(const void *x, const float *dt, const float *A, const float *lam,
                              const float *theta, const void *B, const void *C, const float *D,
                              const float *W_x, const float *W_y, m3_dtype dtype, const m3_bcnorm *norm,
                              const float *h0, const float *prevBx0, const float *angle0, m3_dims d,
                              void *y, float *h_final, float *prevBx_final, float *angle_final,
                              void *workspace, size_t workspace_bytes, void *stream) {
    return chunked_common(x, dt, A, lam, theta, B, C, D, W_x, W_y, dtype, norm, h0, prevBx0, angle0, d, y,
                          h_final, prevBx_final, angle_final, workspace, workspace_bytes, stream, true);
}

m3_status m3_step_decode(const void *x_t, const float *dt_t, const float *A, const float *lam_t,
                         const float *theta_t, const void *B_t, const void *C_t, const float *D,
                         m3_dtype dtype, const m3_bcnorm *norm, m3_dims d, float *h, float *prevBx,
                         float *angle, void *y_t, void *stream) {
    m3_status st;
    if ((st = check_dtype(dtype)) != M3_OK) return st;
    if ((st = check_core_dims(d, false)) != M3_OK) return st;
    int64_t G, K;
    if ((st = resolve_groups(d, G, K)) != M3_OK) return st;
    M3_REQ(A); M3_REQ(D);
    if (d.batch > 0) {
        M3_REQ(x_t); M3_REQ(dt_t); M3_REQ(lam_t); M3_REQ(theta_t); M3_REQ(B_t); M3_REQ(C_t);
        M3_REQ(h); M3_REQ(prevBx); M3_REQ(angle); M3_REQ(y_t);
    }
    NormArgs nrm;
    if ((st = read_norm(norm, nrm)) != M3_OK) return st;
    if (d.batch == 0) return M3_OK;
    DecodeArgs a;
    a.x = x_t; a.B = B_t; a.C = C_t; a.dt = dt_t; a.A = A; a.lam = lam_t; a.theta = theta_t; a.D = D;
    a.nrm = nrm; a.h = h; a.prevBx = prevBx; a.angle = angle; a.y = y_t;
    a.Bt = d.batch; a.H = d.nheads; a.P = d.headdim; a.N = d.dstate; a.G = G; a.K = K;
    return launch_unless_injected([&] { return launch_decode(a, dtype, (cudaStream_t)stream); });
}

namespace {
// Shared validation of the rank-R decode entry points.
m3_status decode_gen(const void *x_t, const float *dt_t, const float *A, const float *lam_t, const float *theta_t,
                     const void *B_t, const void *C_t, const float *D, const float *W_x, const float *W_y,
                     m3_dtype dtype, const m3_bcnorm *norm, m3_dims d, float *h, float *prevBx, float *b_prev,
                     float *x_prev, float *angle, void *y_t, void *stream, bool factored) {
    m3_status st;
    if ((st = check_dtype(dtype)) != M3_OK) return st;
    if ((st = check_core_dims(d, false)) != M3_OK) return st;
    int64_t G, K;
    if ((st = resolve_groups(d, G, K)) != M3_OK) return st;
    if (d.rank < 1) return M3_ERR_INVALID_ARG;
    if (d.rank > kMaxRank || d.headdim % 4) return M3_ERR_UNSUPPORTED;
    M3_REQ(A); M3_REQ(D);
    M3_OPT(W_x); M3_OPT(W_y);
    if (d.batch > 0) {
        M3_REQ(x_t); M3_REQ(dt_t); M3_REQ(lam_t); M3_REQ(theta_t); M3_REQ(B_t); M3_REQ(C_t);
        M3_REQ(h); M3_REQ(angle); M3_REQ(y_t);
        if (factored) { M3_REQ(b_prev); M3_REQ(x_prev); }
        else M3_REQ(prevBx);
    }
    NormArgs nrm;
    if ((st = read_norm(norm, nrm)) != M3_OK) return st;
    if (d.batch == 0) return M3_OK;
    DecodeArgs a;
    a.x = x_t; a.B = B_t; a.C = C_t; a.dt = dt_t; a.A = A; a.lam = lam_t; a.theta = theta_t; a.D = D;
    a.nrm = nrm; a.h = h; a.prevBx = prevBx; a.angle = angle; a.y = y_t;
    a.Bt = d.batch; a.H = d.nheads; a.P = d.headdim; a.N = d.dstate; a.G = G; a.K = K;
    a.Wx = W_x; a.Wy = W_y; a.bprev = b_prev; a.xprev = x_prev; a.R = d.rank;
    return launch_unless_injected([&] { return launch_decode_gen(a, dtype, factored, (cudaStream_t)stream); });
}
}  // namespace

m3_status m3_mimo_step_decode(const void *x_t, const float *dt_t, const float *A, const float *lam_t,
                              const float *theta_t, const void *B_t, const void *C_t, const float *D,
                              const float *W_x, const float *W_y, m3_dtype dtype, const m3_bcnorm *norm,
                              m3_dims d, float *h, float *prevBx, float *angle, void *y_t, void *stream) {
    return decode_gen(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, W_x, W_y, dtype, norm, d, h, prevBx, nullptr,
                      nullptr, angle, y_t, stream, false);
}

m3_status m3_step_decode_factored(const void *x_t, const float *dt_t, const float *A, const float *lam_t,
                                  const float *theta_t, const void *B_t, const void *C_t, const float *D,
                                  const float *W_x, const float *W_y, m3_dtype dtype, const m3_bcnorm *norm,
                                  m3_dims d, float *h, float *b_prev, float *x_prev, float *angle, void *y_t,
                                  void *stream) {
    return decode_gen(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, W_x, W_y, dtype, norm, d, h, nullptr, b_prev,
                      x_prev, angle, y_t, stream, true);
}

m3_status m3_chunked_bwd(const void *x, const float *dt, const float *A, const float *lam, const float *theta,
                         const void *B, const void *C, const float *D, const float *W_x, const float *W_y,
                         m3_dtype dtype, const m3_bcnorm *norm, const float *h0, const float *prevBx0,
                         const float *angle0, m3_dims d, const void *dy, const float *dh_final,
                         const float *dprevBx_final, const float *dangle_final, const m3_grads *grads,
                         void *workspace, size_t workspace_bytes, void *stream) {
    m3_status st;
    if ((st = check_dtype(dtype)) != M3_OK) return st;
    if ((st = check_core_dims(d, true)) != M3_OK) return st;
    if (d.chunk < 1 || d.rank < 0 || !grads) return M3_ERR_INVALID_ARG;
    int64_t G, K;
    if ((st = resolve_groups(d, G, K)) != M3_OK) return st;
    const bool mimo = d.rank > 1 || W_x || W_y;
    const int64_t R = d.rank > 1 ? d.rank : 1;
    if (R > kMaxRank) return M3_ERR_UNSUPPORTED;
    M3_REQ(A); M3_REQ(D);
    const bool have_tokens = d.batch > 0 && d.seqlen > 0;
    if (have_tokens) {
        M3_REQ(x); M3_REQ(dt); M3_REQ(lam); M3_REQ(theta); M3_REQ(B); M3_REQ(C); M3_REQ(dy);
    } else {
        M3_OPT(x); M3_OPT(dt); M3_OPT(lam); M3_OPT(theta); M3_OPT(B); M3_OPT(C); M3_OPT(dy);
    }
    M3_OPT(W_x); M3_OPT(W_y); M3_OPT(h0); M3_OPT(prevBx0); M3_OPT(angle0);
    M3_OPT(dh_final); M3_OPT(dprevBx_final); M3_OPT(dangle_final); M3_OPT(workspace);
    const m3_grads &g = *grads;
    M3_OPT(g.dx); M3_OPT(g.ddt); M3_OPT(g.dA); M3_OPT(g.dlam); M3_OPT(g.dtheta); M3_OPT(g.dB); M3_OPT(g.dC);
    M3_OPT(g.dD); M3_OPT(g.dW_x); M3_OPT(g.dW_y); M3_OPT(g.dnormw_B); M3_OPT(g.dnormw_C); M3_OPT(g.dbias_B);
    M3_OPT(g.dbias_C); M3_OPT(g.dh0); M3_OPT(g.dprevBx0); M3_OPT(g.dangle0);
    NormArgs nrm;
    if ((st = read_norm(norm, nrm)) != M3_OK) return st;
    BwdArgs a{};
    a.x = x; a.B = B; a.C = C; a.dy = dy;
    a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.D = D; a.Wx = W_x; a.Wy = W_y;
    a.h0 = h0; a.prevBx0 = prevBx0; a.angle0 = angle0;
    a.dh = dh_final; a.du = dprevBx_final; a.da = dangle_final;
    a.nrm = nrm;
    a.dx = g.dx; a.ddt = g.ddt; a.dA = g.dA; a.dlam = g.dlam; a.dtheta = g.dtheta; a.dB = g.dB; a.dC = g.dC;
    a.dD = g.dD; a.dWx = g.dW_x; a.dWy = g.dW_y; a.dwB = g.dnormw_B; a.dwC = g.dnormw_C; a.dbB = g.dbias_B;
    a.dbC = g.dbias_C; a.dh0 = g.dh0; a.du0 = g.dprevBx0; a.da0 = g.dangle0;
    a.Bt = d.batch; a.T = d.seqlen; a.H = d.nheads; a.P = d.headdim; a.N = d.dstate; a.R = R; a.G = G; a.K = K;
    const int q = bwd_chunk(a.P, a.N, R, K, d.chunk);
    if (q < 1) return M3_ERR_UNSUPPORTED;
    const size_t need = m3_workspace_bytes(mimo ? M3_WS_BWD_MIMO : M3_WS_BWD_SISO, d, dtype);
    if (need > 0 && (!workspace || workspace_bytes < need)) return M3_ERR_WORKSPACE;
    a.Q = q;
    a.ws = static_cast<float *>(workspace);
    if (d.batch == 0) return M3_OK;
    return launch_unless_injected([&] { return launch_scan_bwd(a, dtype, (cudaStream_t)stream); });
}

}  // extern "C"
