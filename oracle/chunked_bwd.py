"""fp64 chunked form of the scan's backward, SISO and rank R (numpy).

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

Rank R (TorchMamba README, "Math notes": rank-R update on a shared (N,P)
state; App. C per-head expand/contract vectors) is the same walk over rows
(token i, rank r): X_{i,r} = W_x[r] * x_i, the row mask is M[i,j] for every
rank pair, dY_{i,r} = W_y[r] * dy_i, and y_i = sum_r W_y[r] * Y_{i,r} + D x_i.

Scope: SISO and rank R, grouped B/C and partial RoPE, initial states and
final-state adjoints; no QkNorm or bias (those are pinned through the loop
alone).
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


def _lane(x, dt, A, lam, th, B, C, Wx, Wy, D, dy, Q, h0, u0, a0, dh, du, da):
    """One (b, h) lane.  B, C (T, R, N); Wx, Wy (R, P)."""
    T, P = x.shape
    R, N = B.shape[1], B.shape[2]
    phi = a0[None, :] + np.cumsum(dt[:, None] * th, axis=0)
    phr = np.repeat(phi, R, axis=0)                       # every rank turns by the token's angle
    Bb = _rotate(B.reshape(T * R, N), phr)                # rows (t, r)
    Cb = _rotate(C.reshape(T * R, N), phr)
    Xr = (Wx[None] * x[:, None, :]).reshape(T * R, P)
    Dyr = (Wy[None] * dy[:, None, :]).reshape(T * R, P)
    la = dt * A
    gam = lam * dt
    sg = np.zeros(T)
    sg[:-1] = (1.0 - lam[1:]) * dt[1:]
    w = gam + sg
    sg_m1 = (1.0 - lam[0]) * dt[0]
    nch = (T + Q - 1) // Q
    bounds = [(c * Q, min(T, (c + 1) * Q)) for c in range(nch)]
    rows = lambda v: np.repeat(v, R)
    tok = lambda v, n: v.reshape(n, R).sum(axis=1)        # sum a per-row value over each token's ranks

    # forward: the shifted state entering every chunk
    gin = []
    g = h0 + sg_m1 * u0
    for s0, s1 in bounds:
        gin.append(g)
        cum = np.cumsum(la[s0:s1])
        es = np.exp(cum[-1] - cum)
        g = np.exp(cum[-1]) * g + Bb[s0 * R:s1 * R].T @ (rows(es * w[s0:s1])[:, None] * Xr[s0 * R:s1 * R])

    dXr = np.zeros_like(Xr)
    dBb = np.zeros_like(Bb)
    dCb = np.zeros_like(Cb)
    dWy = np.zeros((R, P))
    dla = np.zeros(T)
    dw = np.zeros(T)
    dgam = np.zeros(T)
    dphi = np.zeros_like(phi)
    # the final states: h_final = g after the last token (sg_{T-1} = 0),
    # prevBx_final = sum_r Bbar_{T-1,r} X_{T-1,r}^T, angle_final = phi_{T-1}
    Gout = dh.copy()
    last = slice((T - 1) * R, T * R)
    dBb[last] += Xr[last] @ du.T
    dXr[last] += Bb[last] @ du
    dphi[T - 1] += da

    for c in reversed(range(nch)):
        s0, s1 = bounds[c]
        n = s1 - s0
        rs = slice(s0 * R, s1 * R)
        cum = np.cumsum(la[s0:s1])
        ce = cum[-1]
        ec, es = np.exp(cum), np.exp(ce - cum)
        Cc, Bc, Xc, Dc = Cb[rs], Bb[rs], Xr[rs], Dyr[rs]
        wc, gc = w[s0:s1], gam[s0:s1]
        gi = gin[c]
        dcum = np.zeros(n)
        # token mask and its row expansion (every rank pair of a token pair)
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        low = jj < ii
        E = np.where(low, np.exp(np.where(low, cum[:, None] - cum[None, :], 0.0)), 0.0)
        M = E * wc[None, :] + np.diag(gc)
        Mr = np.kron(M, np.ones((R, R)))
        S = Cc @ Bc.T                                    # Cbar_(i,r) . Bbar_(j,r')
        # the per-rank outputs (for the W_y gradient)
        Y = rows(ec)[:, None] * (Cc @ gi) + (Mr * S) @ Xc
        dWy += (Y.reshape(n, R, P) * dy[s0:s1, None, :]).sum(axis=0)
        # inter-chunk output term e^{cum_i} Cbar_(i,r)^T g_in
        GD = Dc @ gi.T
        dCc = rows(ec)[:, None] * GD
        dcum += ec * tok(np.sum(Cc * GD, axis=1), n)
        dgin = Cc.T @ (rows(ec)[:, None] * Dc)
        # intra-chunk term
        V = Dc @ Xc.T                                    # dY_(i,r) . X_(j,r')
        dXc = (Mr * S).T @ Dc
        dCc = dCc + (Mr * V) @ Bc
        dBc = (Mr * V).T @ Cc
        dM = (S * V).reshape(n, R, n, R).sum(axis=(1, 3))
        t1 = np.where(low, dM * M, 0.0)
        dcum += t1.sum(axis=1) - t1.sum(axis=0)
        dwc = (dM * E).sum(axis=0)
        dgc = np.diag(dM).copy()
        # chunk-state term e^{cum_end - cum_j} w_j Bbar_(j,r) X_(j,r)^T and e^{cum_end} g_in
        BG = Bc @ Gout
        GX = Xc @ Gout.T
        sc = rows(es * wc)
        dXc = dXc + sc[:, None] * BG
        dBc = dBc + sc[:, None] * GX
        t2 = tok(np.sum(Xc * BG, axis=1), n)
        dwc = dwc + es * t2
        des = wc * t2 * es
        dcum[-1] += np.sum(des) + np.exp(ce) * np.sum(gi * Gout)
        dcum -= des
        dgin = dgin + np.exp(ce) * Gout
        dla[s0:s1] = np.cumsum(dcum[::-1])[::-1]
        dXr[rs] += dXc
        dBb[rs] += dBc
        dCb[rs] += dCc
        dw[s0:s1] = dwc
        dgam[s0:s1] = dgc
        Gout = dgin

    # X_(t,r) = W_x[r] x_t and y_t = sum_r W_y[r] Y_(t,r) + D x_t
    dX3 = dXr.reshape(T, R, P)
    dx = (Wx[None] * dX3).sum(axis=1) + D * dy
    dWx = (x[:, None, :] * dX3).sum(axis=0)
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
    # rotation: Bbar = R(phi) B per rank, phi_t = angle0 + sum_{k<=t} dt_k theta_k
    K = phi.shape[1]
    dB = _rotate(dBb, phr, inverse=True).reshape(T, R, N)
    dC = _rotate(dCb, phr, inverse=True).reshape(T, R, N)
    cross = (Bb[:, 0:2 * K:2] * dBb[:, 1:2 * K:2] - Bb[:, 1:2 * K:2] * dBb[:, 0:2 * K:2]
             + Cb[:, 0:2 * K:2] * dCb[:, 1:2 * K:2] - Cb[:, 1:2 * K:2] * dCb[:, 0:2 * K:2])
    dphi += cross.reshape(T, R, K).sum(axis=1)
    rc = np.cumsum(dphi[::-1], axis=0)[::-1]
    dth = dt[:, None] * rc
    ddt += np.sum(th * rc, axis=1)
    da0 = rc[0]
    dD = np.sum(dy * x)
    return dict(dx=dx, ddt=ddt, dA=dA, dlam=dlam, dtheta=dth, dB=dB, dC=dC, dD=dD, dWx=dWx, dWy=dWy,
                dh0=dh0, dprevBx0=du0, dangle0=da0)


def chunked_bwd(x, dt, A, lam, theta, B, C, D, dy, chunk, Wx=None, Wy=None, h0=None, prevBx0=None, angle0=None,
                dh=None, dprevBx=None, dangle=None):
    """Gradients of <dy, y> + <dh, h_final> + <dprevBx, prevBx_final> +
    <dangle, angle_final> by the chunked reverse walk, in fp64.  Layouts as
    ``loop_bwd``: x, dy (Bt,T,H,P); dt, lam (Bt,T,H); A, D (H); theta
    (Bt,T,H,K); B, C (Bt,T,G,N) for SISO or (Bt,T,G,R,N) for rank R; Wx, Wy
    (H,R,P) or None for ones; states (Bt,H,N,P) and (Bt,H,K).  ``chunk``
    counts tokens.  T >= 1.  Returns ``loop_bwd``'s keys for these inputs
    (dWx, dWy only with a rank axis)."""
    x, dt, lam, theta, B, C, dy = (np.asarray(a, dtype=np.float64) for a in (x, dt, lam, theta, B, C, dy))
    A, D = np.asarray(A, dtype=np.float64), np.asarray(D, dtype=np.float64)
    mimo = B.ndim == 5
    if not mimo:
        B, C = B[:, :, :, None, :], C[:, :, :, None, :]
    Bt, T, H, P = x.shape
    G, R, N, K = B.shape[2], B.shape[3], B.shape[4], theta.shape[3]
    if T < 1 or chunk < 1 or H % G or 2 * K > N:
        raise ValueError("bad sizes")
    z = lambda shape, a: np.zeros(shape) if a is None else np.asarray(a, dtype=np.float64)
    h0, prevBx0, dh, dprevBx = (z((Bt, H, N, P), a) for a in (h0, prevBx0, dh, dprevBx))
    angle0, dangle = z((Bt, H, K), angle0), z((Bt, H, K), dangle)
    Wx = np.ones((H, R, P)) if Wx is None else np.asarray(Wx, dtype=np.float64)
    Wy = np.ones((H, R, P)) if Wy is None else np.asarray(Wy, dtype=np.float64)
    out = dict(dx=np.zeros_like(x), ddt=np.zeros_like(dt), dA=np.zeros(H), dlam=np.zeros_like(lam),
               dtheta=np.zeros_like(theta), dB=np.zeros_like(B), dC=np.zeros_like(C), dD=np.zeros(H),
               dWx=np.zeros((H, R, P)), dWy=np.zeros((H, R, P)), dh0=np.zeros((Bt, H, N, P)),
               dprevBx0=np.zeros((Bt, H, N, P)), dangle0=np.zeros((Bt, H, K)))
    for b in range(Bt):
        for h in range(H):
            g = h // (H // G)
            r = _lane(x[b, :, h], dt[b, :, h], A[h], lam[b, :, h], theta[b, :, h], B[b, :, g], C[b, :, g],
                      Wx[h], Wy[h], D[h], dy[b, :, h], chunk, h0[b, h], prevBx0[b, h], angle0[b, h], dh[b, h],
                      dprevBx[b, h], dangle[b, h])
            for k in ("dx", "ddt", "dlam", "dtheta"):
                out[k][b, :, h] = r[k]
            out["dB"][b, :, g] += r["dB"]
            out["dC"][b, :, g] += r["dC"]
            for k in ("dA", "dD", "dWx", "dWy"):
                out[k][h] += r[k]
            for k in ("dh0", "dprevBx0", "dangle0"):
                out[k][b, h] = r[k]
    if not mimo:
        out["dB"], out["dC"] = out["dB"][:, :, :, 0], out["dC"][:, :, :, 0]
        del out["dWx"], out["dWy"]
    return out
