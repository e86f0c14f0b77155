"""fp64 chunked form of the SISO scan's backward (numpy).

TEST INFRASTRUCTURE ONLY, like the rest of this package: it is a second
formulation of the gradients, checked against the loop's reverse sweep
(``loop_bwd``, itself pinned by finite differences), so that the chunked
adjoint that a blocked kernel computes is written out here in plain form.

The forward it differentiates is the chunked form of the trapezoidal
recurrence (dotLLM pull request, "Stage A: Mamba3SelectiveScan" and the
streaming-decode comment on shifted_gamma and the boundary fold; TorchMamba
README, "Math notes": Mamba-2 chunkwise intra-chunk quadratic part plus an
inter-chunk carry, Props. 2-4 for the rotation).  With
sg_t = (1 - lam_{t+1}) dt_{t+1} (0 at the last token), w_t = gamma_t + sg_t
and U_t = Bbar_t x_t^T, the shifted state g_t = h_t + sg_t U_t obeys
g_t = alpha_t g_{t-1} + w_t U_t from g_{-1} = h0 + (1 - lam_0) dt_0 prevBx0.
Inside a chunk, with cum_i the running sum of log alpha from its start:

    y_i   = e^{cum_i} Cbar_i^T g_in + sum_{j<=i} M[i,j] (Cbar_i . Bbar_j) x_j + D x_i
    g_out = e^{cum_end} g_in + sum_j e^{cum_end - cum_j} w_j Bbar_j x_j^T
    M[i,j] = e^{cum_i - cum_j} w_j (j < i),  gamma_i (j = i)

The backward walks the chunks in reverse with the adjoint Gout of g_out
(the adjoint of h_final for the last chunk), and per chunk:

    dCbar_i += e^{cum_i} g_in dy_i + sum_j M[i,j] (dy_i . x_j) Bbar_j
    dBbar_j += sum_i M[i,j] (dy_i . x_j) Cbar_i + e^{cum_end - cum_j} w_j Gout x_j
    dx_j    += sum_i M[i,j] (Cbar_i . Bbar_j) dy_i + e^{cum_end - cum_j} w_j Bbar_j^T Gout
    dg_in    = sum_i e^{cum_i} Cbar_i dy_i^T + e^{cum_end} Gout

and the decay, weight and angle adjoints follow from the same terms.

Scope: SISO (B, C without a rank axis), grouped B/C and partial RoPE,
initial states and final-state adjoints; no QkNorm or bias (those are
pinned through the loop alone).
"""
import numpy as np


def _rotate(v, phi, inverse=False):
    """Rotate the first K pairs (2i, 2i+1) of v (T, N) by +phi (T, K)."""
    K = phi.shape[1]
    out = v.copy()
    c, s = np.cos(phi), np.sin(phi)
    if inverse:
        s = -s
    e, o = v[:, 0:2 * K:2], v[:, 1:2 * K:2]
    out[:, 0:2 * K:2] = c * e - s * o
    out[:, 1:2 * K:2] = s * e + c * o
    return out


def _lane(x, dt, A, lam, th, B, C, D, dy, Q, h0, u0, a0, dh, du, da):
    T, P = x.shape
    N = B.shape[1]
    phi = a0[None, :] + np.cumsum(dt[:, None] * th, axis=0)
    Bb, Cb = _rotate(B, phi), _rotate(C, phi)
    la = dt * A
    gam = lam * dt
    sg = np.zeros(T)
    sg[:-1] = (1.0 - lam[1:]) * dt[1:]
    w = gam + sg
    sg_m1 = (1.0 - lam[0]) * dt[0]
    nch = (T + Q - 1) // Q
    bounds = [(c * Q, min(T, (c + 1) * Q)) for c in range(nch)]

    # forward: the shifted state entering every chunk
    gin = []
    g = h0 + sg_m1 * u0
    for s0, s1 in bounds:
        gin.append(g)
        cum = np.cumsum(la[s0:s1])
        es = np.exp(cum[-1] - cum)
        g = np.exp(cum[-1]) * g + Bb[s0:s1].T @ ((es * w[s0:s1])[:, None] * x[s0:s1])

    dx = D * dy
    dBb = np.zeros_like(B)
    dCb = np.zeros_like(C)
    dla = np.zeros(T)
    dw = np.zeros(T)
    dgam = np.zeros(T)
    dphi = np.zeros_like(phi)
    # the final states: h_final = g after the last token (sg_{T-1} = 0),
    # prevBx_final = U_{T-1}, angle_final = phi_{T-1}
    Gout = dh.copy()
    dBb[T - 1] += du @ x[T - 1]
    dx[T - 1] += du.T @ Bb[T - 1]
    dphi[T - 1] += da

    for c in reversed(range(nch)):
        s0, s1 = bounds[c]
        n = s1 - s0
        cum = np.cumsum(la[s0:s1])
        ce = cum[-1]
        ec, es = np.exp(cum), np.exp(ce - cum)
        Cc, Bc, Xc, Dc = Cb[s0:s1], Bb[s0:s1], x[s0:s1], dy[s0:s1]
        wc, gc = w[s0:s1], gam[s0:s1]
        gi = gin[c]
        dcum = np.zeros(n)
        # inter-chunk output term e^{cum_i} Cbar_i^T g_in
        GD = Dc @ gi.T                                   # row i: g_in dy_i
        dCc = ec[:, None] * GD
        dcum += ec * np.sum(Cc * GD, axis=1)
        dgin = Cc.T @ (ec[:, None] * Dc)
        # intra-chunk term
        S = Cc @ Bc.T                                    # Cbar_i . Bbar_j
        V = Dc @ Xc.T                                    # dy_i . x_j
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        low = jj < ii
        E = np.where(low, np.exp(np.where(low, cum[:, None] - cum[None, :], 0.0)), 0.0)
        M = E * wc[None, :] + np.diag(gc)
        dxc = (M * S).T @ Dc
        dCc = dCc + (M * V) @ Bc
        dBc = (M * V).T @ Cc
        dM = S * V
        t1 = np.where(low, dM * M, 0.0)
        dcum += t1.sum(axis=1) - t1.sum(axis=0)
        dwc = (dM * E).sum(axis=0)
        dgc = np.diag(dM).copy()
        # chunk-state term e^{cum_end - cum_j} w_j Bbar_j x_j^T and e^{cum_end} g_in
        BG = Bc @ Gout                                   # row j: Bbar_j^T Gout
        GX = Xc @ Gout.T                                 # row j: Gout x_j
        sc = es * wc
        dxc = dxc + sc[:, None] * BG
        dBc = dBc + sc[:, None] * GX
        t2 = np.sum(Xc * BG, axis=1)
        dwc = dwc + es * t2
        des = wc * t2 * es
        dcum[-1] += np.sum(des) + np.exp(ce) * np.sum(gi * Gout)
        dcum -= des
        dgin = dgin + np.exp(ce) * Gout
        dla[s0:s1] = np.cumsum(dcum[::-1])[::-1]
        dx[s0:s1] += dxc
        dBb[s0:s1] += dBc
        dCb[s0:s1] += dCc
        dw[s0:s1] = dwc
        dgam[s0:s1] = dgc
        Gout = dgin

    # g_{-1} = h0 + sg_{-1} prevBx0
    dh0 = Gout
    du0 = sg_m1 * Gout
    dsg_m1 = np.sum(u0 * Gout)
    # la = dt A; gamma = lam dt; sg_t = (1 - lam_{t+1}) dt_{t+1}; w = gamma + sg
    ddt = A * dla
    dA = np.sum(dt * dla)
    dgam = dgam + dw
    ddt += lam * dgam
    dlam = dt * dgam
    ddt[1:] += (1.0 - lam[1:]) * dw[:-1]
    dlam[1:] -= dt[1:] * dw[:-1]
    ddt[0] += (1.0 - lam[0]) * dsg_m1
    dlam[0] -= dt[0] * dsg_m1
    # rotation: Bbar = R(phi) B, phi_t = angle0 + sum_{k<=t} dt_k theta_k
    K = phi.shape[1]
    dB, dC = _rotate(dBb, phi, inverse=True), _rotate(dCb, phi, inverse=True)
    dphi += (Bb[:, 0:2 * K:2] * dBb[:, 1:2 * K:2] - Bb[:, 1:2 * K:2] * dBb[:, 0:2 * K:2]
             + Cb[:, 0:2 * K:2] * dCb[:, 1:2 * K:2] - Cb[:, 1:2 * K:2] * dCb[:, 0:2 * K:2])
    rc = np.cumsum(dphi[::-1], axis=0)[::-1]
    dth = dt[:, None] * rc
    ddt += np.sum(th * rc, axis=1)
    da0 = rc[0]
    dD = np.sum(dy * x)
    return dict(dx=dx, ddt=ddt, dA=dA, dlam=dlam, dtheta=dth, dB=dB, dC=dC, dD=dD, dh0=dh0,
                dprevBx0=du0, dangle0=da0)


def siso_chunked_bwd(x, dt, A, lam, theta, B, C, D, dy, chunk, h0=None, prevBx0=None, angle0=None, dh=None,
                     dprevBx=None, dangle=None):
    """Gradients of <dy, y> + <dh, h_final> + <dprevBx, prevBx_final> +
    <dangle, angle_final> by the chunked reverse walk, in fp64.  Layouts as
    ``loop_bwd``: x, dy (Bt,T,H,P); dt, lam (Bt,T,H); A, D (H); theta
    (Bt,T,H,K); B, C (Bt,T,G,N); states (Bt,H,N,P) and (Bt,H,K).  T >= 1.
    Returns the dict of ``loop_bwd``'s keys for these inputs."""
    x, dt, lam, theta, B, C, dy = (np.asarray(a, dtype=np.float64) for a in (x, dt, lam, theta, B, C, dy))
    A, D = np.asarray(A, dtype=np.float64), np.asarray(D, dtype=np.float64)
    Bt, T, H, P = x.shape
    G, N, K = B.shape[2], B.shape[3], theta.shape[3]
    if T < 1 or chunk < 1 or H % G or 2 * K > N:
        raise ValueError("bad sizes")
    z = lambda shape, a: np.zeros(shape) if a is None else np.asarray(a, dtype=np.float64)
    h0, prevBx0, dh, dprevBx = (z((Bt, H, N, P), a) for a in (h0, prevBx0, dh, dprevBx))
    angle0, dangle = z((Bt, H, K), angle0), z((Bt, H, K), dangle)
    out = dict(dx=np.zeros_like(x), ddt=np.zeros_like(dt), dA=np.zeros(H), dlam=np.zeros_like(lam),
               dtheta=np.zeros_like(theta), dB=np.zeros_like(B), dC=np.zeros_like(C), dD=np.zeros(H),
               dh0=np.zeros((Bt, H, N, P)), dprevBx0=np.zeros((Bt, H, N, P)), dangle0=np.zeros((Bt, H, K)))
    for b in range(Bt):
        for h in range(H):
            g = h // (H // G)
            r = _lane(x[b, :, h], dt[b, :, h], A[h], lam[b, :, h], theta[b, :, h], B[b, :, g], C[b, :, g], D[h],
                      dy[b, :, h], chunk, h0[b, h], prevBx0[b, h], angle0[b, h], dh[b, h], dprevBx[b, h],
                      dangle[b, h])
            out["dx"][b, :, h] = r["dx"]
            out["ddt"][b, :, h] = r["ddt"]
            out["dlam"][b, :, h] = r["dlam"]
            out["dtheta"][b, :, h] = r["dtheta"]
            out["dB"][b, :, g] += r["dB"]
            out["dC"][b, :, g] += r["dC"]
            out["dA"][h] += r["dA"]
            out["dD"][h] += r["dD"]
            out["dh0"][b, h] = r["dh0"]
            out["dprevBx0"][b, h] = r["dprevBx0"]
            out["dangle0"][b, h] = r["dangle0"]
    return out
