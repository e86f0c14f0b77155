"""Pins of the fp64 oracle against facts other than itself (CPU only).

Each pin restates what the pages fix in a formulation independent of the
oracle's code:

* complex SSM: the data-dependent RoPE on B and C is the real form of a
  complex diagonal SSM whose transition carries the rotation
  (TorchMamba README, "Math notes": Props. 2-4; Mamba-3-Lite "Model
  reference": the effective step exp(softplus(dt) A) with complex A, real part
  decay, imaginary part rotation);
* matrix form: y = (L o (C B^T)) x with L = 1SS(alpha) @ Band -- a matrix
  product, not a Hadamard product (TorchMamba README, "Math notes", Eq. 7);
* closed form of the recurrence with constant inputs;
* reductions Mamba-3 SISO -> Mamba-2 SSD at lam = 1, theta = 0 and
  Mamba-2 -> Mamba-1 S6 (exponential-Euler) at P = 1 (TorchMamba README,
  "Models" and "Math notes");
* MIMO: R = 1 equals SISO; MIMO equals R stacked SISO scans / R^2 SISO calls
  (TorchMamba README, "Math notes", MIMO; Eqs. 12-14);
* split schedules: prefill + decode reproduces the one-shot scan (dotLLM pull
  request, "Mamba-3 streaming decode" and "MIMO streaming decode": schedules
  2+2+2, 1+1+1+1+1+1, 3+3, 4+2, 2+4, 1+2+3, 5+1);
* MIMO decode steps, and decode steps on the factored previous-input state
  (previous token's rotated B per rank and its x), reproduce the one-shot
  MIMO scan (dotLLM pull request, "MIMO streaming decode"; TorchMamba README,
  "Models": cache of angle, ssm, x_prev, b_prev);
* grouped B/C equals per-head B/C repeated over each group's heads, and
  partial RoPE equals full RoPE with theta zero beyond the first K pairs
  (TorchMamba README, "Models": n_groups; dotLLM pull request, real-checkpoint
  run: num_rope_angles 32 of d_state 128);
* chunked fp64 form equals the loop (ats-v2 README, "Mamba uses a chunked
  parallel scan": exact at float64);
* rotation invariance and the trapezoid weights' sum.

Tolerances follow the TorchMamba README's fp64 convention (rtol 1e-10,
atol 1e-12).
"""
import numpy as np
import pytest

RTOL, ATOL = 1e-10, 1e-12


def rnd_inputs(rng, Bt=2, T=9, H=3, P=4, N=6, R=1, dt_shift=-1.0):
    sp = lambda v: np.log1p(np.exp(v))
    x = rng.standard_normal((Bt, T, H, P))
    dt = sp(rng.standard_normal((Bt, T, H)) + dt_shift)
    A = -np.exp(rng.uniform(0, 1, H))
    lam = 1 / (1 + np.exp(-rng.standard_normal((Bt, T, H))))
    theta = rng.uniform(-np.pi / 2, np.pi / 2, (Bt, T, H, N // 2))
    shp = (Bt, T, H, N) if R == 1 else (Bt, T, H, R, N)
    B = rng.standard_normal(shp) / np.sqrt(N)
    C = rng.standard_normal(shp) / np.sqrt(N)
    D = rng.standard_normal(H)
    return dict(x=x, dt=dt, A=A, lam=lam, theta=theta, B=B, C=C, D=D)


def close(a, b, rtol=RTOL, atol=ATOL):
    np.testing.assert_allclose(a, b, rtol=rtol, atol=atol)


# ----------------------------------------------------------------------------
# complex diagonal SSM (no rotation of B/C at all)
# ----------------------------------------------------------------------------
def complex_ssm(inp):
    """Complex-state form: per pair i the state is complex, the transition is
    exp(dt (A - i theta)), and the exponential-trapezoidal rule applies the
    full complex transition to the previous-input term."""
    x, dt, A, lam, theta, B, C, D = (inp[k] for k in "x dt A lam theta B C D".split())
    Bt, T, H, P = x.shape
    N = B.shape[-1]
    zB = B[..., 0::2] + 1j * B[..., 1::2]
    zC = C[..., 0::2] + 1j * C[..., 1::2]
    y = np.zeros_like(x)
    hfin = np.zeros((Bt, H, N // 2, P), complex)
    for b in range(Bt):
        for h in range(H):
            hc = np.zeros((N // 2, P), complex)
            prev = np.zeros((N // 2, P), complex)
            for t in range(T):
                Abar = np.exp(dt[b, t, h] * (A[h] - 1j * theta[b, t, h]))
                cur = np.outer(zB[b, t, h], x[b, t, h])
                hc = (Abar[:, None] * hc + (1 - lam[b, t, h]) * dt[b, t, h] * Abar[:, None] * prev
                      + lam[b, t, h] * dt[b, t, h] * cur)
                prev = cur
                y[b, t, h] = np.real(np.conj(zC[b, t, h])[:, None] * hc).sum(0) + D[h] * x[b, t, h]
            hfin[b, h] = hc
    return y, hfin


def test_complex_ssm_equivalence(oracle_mod):
    rng = np.random.default_rng(1)
    inp = rnd_inputs(rng)
    y, hf, ub, ang = oracle_mod.siso_loop(**inp)
    yc, hc = complex_ssm(inp)
    close(y, yc)
    # the oracle's state is the complex state expressed in the rotated frame
    G = hf[:, :, 0::2, :] + 1j * hf[:, :, 1::2, :]
    rot = np.exp(1j * ang)[..., None]
    close(G, rot * hc)
    # angle_final = sum_t dt_t theta_t
    close(ang, np.einsum("bth,bthi->bhi", inp["dt"], inp["theta"]))


def test_complex_ssm_equivalence_mimo_r1(oracle_mod):
    rng = np.random.default_rng(2)
    inp = rnd_inputs(rng, R=1)
    B5 = inp["B"][:, :, :, None, :]
    C5 = inp["C"][:, :, :, None, :]
    y, hf, ub, ang = oracle_mod.mimo_loop(**{**inp, "B": B5, "C": C5})
    yc, hc = complex_ssm(inp)
    close(y, yc)


# ----------------------------------------------------------------------------
# matrix (quadratic) form, Eq. 7: L = 1SS(alpha) @ Band
# ----------------------------------------------------------------------------
def test_matrix_form(oracle_mod):
    rng = np.random.default_rng(3)
    inp = rnd_inputs(rng, Bt=1, T=16, H=2, P=3, N=4)
    y, *_ = oracle_mod.siso_loop(**inp)
    al, be, ga = oracle_mod.discretize(inp["dt"], inp["A"], inp["lam"])
    Br, Cr, _ = oracle_mod.rope_bc(inp["B"], inp["C"], inp["theta"], inp["dt"])
    T = 16
    for h in range(2):
        a = al[0, :, h]
        ss = np.zeros((T, T))          # 1-semiseparable: prod_{k=s+1..t} a_k
        for t in range(T):
            for s in range(t + 1):
                ss[t, s] = np.prod(a[s + 1:t + 1])
        band = np.diag(ga[0, :, h]) + np.diag(be[0, 1:, h], -1)
        L = ss @ band
        G = Cr[0, :, h] @ Br[0, :, h].T
        ym = (L * G) @ inp["x"][0, :, h] + inp["D"][h] * inp["x"][0, :, h]
        close(y[0, :, h], ym)


# ----------------------------------------------------------------------------
# closed form with constant inputs and no rotation
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1, 2, 7, 40])
def test_closed_form(oracle_mod, T):
    H, P, N = 1, 3, 4
    rng = np.random.default_rng(4)
    dtv, lamv, Av = 0.3, 0.35, -0.8
    xv = rng.standard_normal(P)
    Bv = rng.standard_normal(N)
    Cv = rng.standard_normal(N)
    inp = dict(x=np.broadcast_to(xv, (1, T, H, P)).copy(), dt=np.full((1, T, H), dtv),
               A=np.array([Av]), lam=np.full((1, T, H), lamv),
               theta=np.zeros((1, T, H, N // 2)), B=np.broadcast_to(Bv, (1, T, H, N)).copy(),
               C=np.broadcast_to(Cv, (1, T, H, N)).copy(), D=np.array([0.5]))
    y, hf, ub, _ = oracle_mod.siso_loop(**inp)
    a = np.exp(dtv * Av)
    b = (1 - lamv) * dtv * a
    g = lamv * dtv
    U = np.outer(Bv, xv)
    for t in range(T):
        ht = a ** t * g * U + (b + g) * U * (1 - a ** t) / (1 - a)
        close(y[0, t, 0], Cv @ ht + 0.5 * xv, rtol=1e-12)
    close(hf[0, 0], a ** (T - 1) * g * U + (b + g) * U * (1 - a ** (T - 1)) / (1 - a), rtol=1e-12)
    close(ub[0, 0], U)


# ----------------------------------------------------------------------------
# reductions
# ----------------------------------------------------------------------------
def mamba2_loop(x, dt, A, B, C, D):
    """Mamba-2 SSD recurrence with dt folded into B:
    h = exp(dt A) h + dt B x^T,  y = C^T h + D x."""
    Bt, T, H, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    hs = np.zeros((Bt, H, N, P))
    for t in range(T):
        a = np.exp(dt[:, t] * A[None, :])                      # (Bt,H)
        hs = a[..., None, None] * hs + (dt[:, t, :, None, None] * B[:, t, :, :, None]
                                        * x[:, t, :, None, :])
        y[:, t] = np.einsum("bhn,bhnp->bhp", C[:, t], hs) + D[None, :, None] * x[:, t]
    return y, hs


def test_reduction_mamba2(oracle_mod):
    rng = np.random.default_rng(5)
    inp = rnd_inputs(rng, Bt=2, T=12, H=3, P=5, N=6)
    inp["lam"] = np.ones_like(inp["lam"])
    inp["theta"] = np.zeros_like(inp["theta"])
    y, hf, ub, _ = oracle_mod.siso_loop(**inp)
    y2, h2 = mamba2_loop(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    close(y, y2)
    close(hf, h2)
    al, be, ga = oracle_mod.discretize(inp["dt"], inp["A"], inp["lam"])
    assert np.all(be == 0.0)
    close(ga, inp["dt"])


def s6_loop(u, delta, a, Bm, Cm, Dv):
    """Mamba-1 selective scan, exponential-Euler: per channel d with scalar
    decay a_d shared over the state axis; B, C shared by all channels."""
    Bt, L, Dch = u.shape
    N = Bm.shape[-1]
    y = np.zeros_like(u)
    hs = np.zeros((Bt, Dch, N))
    for t in range(L):
        hs = np.exp(delta[:, t, :, None] * a[None, :, None]) * hs + \
            delta[:, t, :, None] * Bm[:, t, None, :] * u[:, t, :, None]
        y[:, t] = (hs * Cm[:, t, None, :]).sum(-1) + Dv * u[:, t]
    return y


def test_reduction_mamba1_p1(oracle_mod):
    rng = np.random.default_rng(6)
    Bt, L, Dch, N = 2, 10, 5, 4
    u = rng.standard_normal((Bt, L, Dch))
    delta = np.log1p(np.exp(rng.standard_normal((Bt, L, Dch)) - 1))
    a = -np.exp(rng.uniform(0, 1, Dch))
    Bm = rng.standard_normal((Bt, L, N))
    Cm = rng.standard_normal((Bt, L, N))
    Dv = rng.standard_normal(Dch)
    ys6 = s6_loop(u, delta, a, Bm, Cm, Dv)
    # channels -> heads with P = 1; B, C broadcast over heads; lam = 1, theta = 0
    inp = dict(x=u[..., None], dt=delta, A=a, lam=np.ones((Bt, L, Dch)),
               theta=np.zeros((Bt, L, Dch, N // 2)),
               B=np.broadcast_to(Bm[:, :, None, :], (Bt, L, Dch, N)).copy(),
               C=np.broadcast_to(Cm[:, :, None, :], (Bt, L, Dch, N)).copy(), D=Dv)
    y, *_ = oracle_mod.siso_loop(**inp)
    close(y[..., 0], ys6)


# ----------------------------------------------------------------------------
# MIMO
# ----------------------------------------------------------------------------
def test_mimo_r1_equals_siso(oracle_mod):
    rng = np.random.default_rng(7)
    inp = rnd_inputs(rng)
    h0 = rng.standard_normal((2, 3, 6, 4))
    u0 = rng.standard_normal((2, 3, 6, 4))
    a0 = rng.uniform(-3, 3, (2, 3, 3))
    s = oracle_mod.siso_loop(**inp, h0=h0, prevBx0=u0, angle0=a0)
    m = oracle_mod.mimo_loop(**{**inp, "B": inp["B"][:, :, :, None], "C": inp["C"][:, :, :, None]},
                             h0=h0, prevBx0=u0, angle0=a0)
    for a, b in zip(s, m):
        np.testing.assert_array_equal(a, b)


def test_mimo_is_r2_siso_calls(oracle_mod):
    rng = np.random.default_rng(8)
    R = 3
    inp = rnd_inputs(rng, Bt=2, T=7, H=2, P=4, N=6, R=R)
    Wx = 1 + 0.3 * rng.standard_normal((2, R, 4))
    Wy = 1 + 0.3 * rng.standard_normal((2, R, 4))
    y, hf, ub, ang = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    D0 = np.zeros_like(inp["D"])
    hsum = np.zeros_like(hf)
    usum = np.zeros_like(ub)
    ysum = np.zeros_like(y)
    for r in range(R):
        xr = inp["x"] * Wx[None, None, :, r, :]
        s = oracle_mod.siso_loop(**{**inp, "x": xr, "B": inp["B"][:, :, :, r], "C": inp["C"][:, :, :, 0],
                                    "D": D0})
        hsum += s[1]
        usum += s[2]
        for rp in range(R):
            yr = oracle_mod.siso_loop(**{**inp, "x": xr, "B": inp["B"][:, :, :, r],
                                         "C": inp["C"][:, :, :, rp], "D": D0})[0]
            ysum += Wy[None, None, :, rp, :] * yr
    ysum += inp["D"][None, None, :, None] * inp["x"]
    close(hf, hsum)
    close(ub, usum)
    close(y, ysum)


# ----------------------------------------------------------------------------
# split schedules: prefill in pieces == one shot
# ----------------------------------------------------------------------------
SCHEDULES = [[6], [2, 2, 2], [1, 1, 1, 1, 1, 1], [3, 3], [4, 2], [2, 4], [1, 2, 3], [5, 1]]


def _run_pieces(fn, inp, sched, bc_keys=("B", "C"), **kw):
    h = u = a = None
    ys = []
    t0 = 0
    for n in sched:
        piece = {k: (v[:, t0:t0 + n] if k in ("x", "dt", "lam", "theta") + bc_keys else v)
                 for k, v in inp.items()}
        y, h, u, a = fn(**piece, h0=h, prevBx0=u, angle0=a, **kw)
        ys.append(y)
        t0 += n
    return np.concatenate(ys, 1), h, u, a


@pytest.mark.parametrize("sched", SCHEDULES)
def test_split_schedules_siso(oracle_mod, sched):
    rng = np.random.default_rng(9)
    inp = rnd_inputs(rng, Bt=2, T=6, H=4, P=4, N=8)
    one = oracle_mod.siso_loop(**inp)
    pcs = _run_pieces(oracle_mod.siso_loop, inp, sched)
    for a, b in zip(one, pcs):
        close(a, b)


@pytest.mark.parametrize("sched", SCHEDULES)
def test_split_schedules_mimo(oracle_mod, sched):
    rng = np.random.default_rng(10)
    inp = rnd_inputs(rng, Bt=1, T=6, H=4, P=4, N=8, R=3)
    Wx = 1 + 0.1 * rng.standard_normal((4, 3, 4))
    Wy = 1 + 0.1 * rng.standard_normal((4, 3, 4))
    one = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    pcs = _run_pieces(oracle_mod.mimo_loop, inp, sched, Wx=Wx, Wy=Wy)
    for a, b in zip(one, pcs):
        close(a, b)


def test_prefill_then_decode_steps(oracle_mod):
    rng = np.random.default_rng(11)
    inp = rnd_inputs(rng, Bt=2, T=17, H=2, P=4, N=6)
    y1, h1, u1, a1 = oracle_mod.siso_loop(**inp)
    k = 9
    pre = {kk: (v[:, :k] if kk in ("x", "dt", "lam", "theta", "B", "C") else v) for kk, v in inp.items()}
    y, h, u, a = oracle_mod.siso_loop(**pre)
    ys = [y]
    for t in range(k, 17):
        yt, h, u, a = oracle_mod.step_decode(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["lam"][:, t],
                                             inp["theta"][:, t], inp["B"][:, t], inp["C"][:, t], inp["D"],
                                             h, u, a)
        ys.append(yt[:, None])
    close(np.concatenate(ys, 1), y1)
    close(h, h1)
    close(u, u1)
    close(a, a1)


# ----------------------------------------------------------------------------
# MIMO decode, and decode on the factored previous-input state (dotLLM pull
# request, "Mamba-3 MIMO streaming decode"; TorchMamba README, "Models": the
# cache carries (angle, ssm, x_prev, b_prev)) == the one-shot MIMO scan
# ----------------------------------------------------------------------------
def _mimo_inputs(rng, Bt, T, H, P, N, R):
    inp = rnd_inputs(rng, Bt=Bt, T=T, H=H, P=P, N=N, R=R)
    if R == 1:   # the factored step takes B, C with an explicit rank axis
        inp["B"], inp["C"] = inp["B"][:, :, :, None], inp["C"][:, :, :, None]
    Wx = 1 + 0.3 * rng.standard_normal((H, R, P))
    Wy = 1 + 0.3 * rng.standard_normal((H, R, P))
    return inp, Wx, Wy


def _tok(inp, t):
    return [inp[k][:, t] for k in ("x", "dt")] + [inp["A"]] + [inp[k][:, t] for k in ("lam", "theta", "B", "C")] + [inp["D"]]


def _outer(bprev, xprev, Wx):
    """prev_Bx rebuilt from its factors: sum_r b_prev[r] (W_x[r] x_prev)^T."""
    return np.einsum("bhrn,hrp,bhp->bhnp", bprev, Wx, xprev)


@pytest.mark.parametrize("R", [1, 3])
def test_factored_decode_from_zero_equals_mimo_loop(oracle_mod, R):
    rng = np.random.default_rng(40 + R)
    Bt, T, H, P, N = 2, 7, 2, 3, 6
    inp, Wx, Wy = _mimo_inputs(rng, Bt, T, H, P, N, R)
    y1, h1, u1, a1 = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    h, bp, xp, a = np.zeros((Bt, H, N, P)), np.zeros((Bt, H, R, N)), np.zeros((Bt, H, P)), np.zeros((Bt, H, N // 2))
    for t in range(T):
        yt, h, bp, xp, a = oracle_mod.step_decode_factored(*_tok(inp, t), h, bp, xp, a, Wx=Wx, Wy=Wy)
        close(yt, y1[:, t])
    close(h, h1)
    close(_outer(bp, xp, Wx), u1)
    close(a, a1)


def test_factored_and_mimo_decode_with_norm_bias_equal_the_loop(oracle_mod):
    """QkNorm gains and per-head biases in the decode steps: factored and full
    state, grouped B/C, partial RoPE, against the one-shot loop."""
    rng = np.random.default_rng(47)
    Bt, T, H, G, P, N, R, K = 2, 5, 4, 2, 3, 8, 2, 3
    inp = _grouped(rng, Bt, T, H, G, P, N, R, K)
    Wx = 1 + 0.3 * rng.standard_normal((H, R, P))
    Wy = 1 + 0.3 * rng.standard_normal((H, R, P))
    nrm = dict(normw_B=1 + 0.2 * rng.standard_normal(N), normw_C=1 + 0.2 * rng.standard_normal(N),
               bias_B=rng.standard_normal((H, R, N)), bias_C=rng.standard_normal((H, R, N)), eps=1e-5)
    y1, h1, u1, a1 = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy, norm=nrm)
    h, u, a = np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N, P)), np.zeros((Bt, H, K))
    hf, bp, xp, af = h.copy(), np.zeros((Bt, H, R, N)), np.zeros((Bt, H, P)), a.copy()
    for t in range(T):
        yt, h, u, a = oracle_mod.mimo_step_decode(*_tok(inp, t), h, u, a, Wx=Wx, Wy=Wy, norm=nrm)
        close(yt, y1[:, t])
        yf, hf, bp, xp, af = oracle_mod.step_decode_factored(*_tok(inp, t), hf, bp, xp, af, Wx=Wx, Wy=Wy,
                                                             norm=nrm)
        close(yf, y1[:, t])
    close(h, h1)
    close(u, u1)
    close(hf, h1)
    close(af, a1)


def test_factored_decode_after_prefill(oracle_mod):
    """Schedule 4 + 3: a prefill by the loop, then decode steps on the factored
    state taken from the prefill's last token (its rotated B and its x)."""
    rng = np.random.default_rng(44)
    Bt, T, H, P, N, R, k = 2, 7, 3, 4, 8, 2, 4
    inp, Wx, Wy = _mimo_inputs(rng, Bt, T, H, P, N, R)
    y1, h1, u1, a1 = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    pre = {kk: (v[:, :k] if kk in ("x", "dt", "lam", "theta", "B", "C") else v) for kk, v in inp.items()}
    _, h, u, a = oracle_mod.mimo_loop(**pre, Wx=Wx, Wy=Wy)
    Br, _, _ = oracle_mod.rope_bc(pre["B"], pre["C"], pre["theta"], pre["dt"])
    bp, xp = Br[:, k - 1], inp["x"][:, k - 1]
    close(_outer(bp, xp, Wx), u)       # the factors rebuild the prefill's prev_Bx
    for t in range(k, T):
        yt, h, bp, xp, a = oracle_mod.step_decode_factored(*_tok(inp, t), h, bp, xp, a, Wx=Wx, Wy=Wy)
        close(yt, y1[:, t])
    close(h, h1)
    close(a, a1)


def test_factored_decode_r1_equals_siso_decode(oracle_mod):
    rng = np.random.default_rng(45)
    Bt, T, H, P, N = 1, 6, 2, 5, 4
    inp = rnd_inputs(rng, Bt=Bt, T=T, H=H, P=P, N=N)
    h, u, a = np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N // 2))
    hf, bp, xp, af = h.copy(), np.zeros((Bt, H, 1, N)), np.zeros((Bt, H, P)), a.copy()
    for t in range(T):
        ys, h, u, a = oracle_mod.step_decode(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["lam"][:, t],
                                             inp["theta"][:, t], inp["B"][:, t], inp["C"][:, t], inp["D"],
                                             h, u, a)
        yf, hf, bp, xp, af = oracle_mod.step_decode_factored(
            inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["lam"][:, t], inp["theta"][:, t],
            inp["B"][:, t, :, None], inp["C"][:, t, :, None], inp["D"], hf, bp, xp, af)
        close(yf, ys)
    close(hf, h)
    close(_outer(bp, xp, np.ones((H, 1, P))), u)


def test_mimo_decode_steps_equal_mimo_loop(oracle_mod):
    rng = np.random.default_rng(46)
    Bt, T, H, P, N, R = 2, 6, 2, 4, 6, 4
    inp, Wx, Wy = _mimo_inputs(rng, Bt, T, H, P, N, R)
    y1, h1, u1, a1 = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    h, u, a = np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N // 2))
    for t in range(T):
        yt, h, u, a = oracle_mod.mimo_step_decode(*_tok(inp, t), h, u, a, Wx=Wx, Wy=Wy)
        close(yt, y1[:, t])
    close(h, h1)
    close(u, u1)
    close(a, a1)


# ----------------------------------------------------------------------------
# grouped B/C (TorchMamba README, "Models": n_groups with H % G == 0; head h
# reads group h // (H / G)) == per-head B/C repeated over each group's heads;
# partial RoPE (dotLLM pull request, real-checkpoint run: num_rope_angles 32
# of d_state 128) == full RoPE with theta zero beyond the first K pairs, and
# as complex numbers only the first K pairs turn
# ----------------------------------------------------------------------------
def _grouped(rng, Bt, T, H, G, P, N, R, K):
    inp = rnd_inputs(rng, Bt=Bt, T=T, H=H, P=P, N=N, R=R)
    shp = (Bt, T, G, N) if R == 1 else (Bt, T, G, R, N)
    inp["B"] = rng.standard_normal(shp) / np.sqrt(N)
    inp["C"] = rng.standard_normal(shp) / np.sqrt(N)
    inp["theta"] = inp["theta"][..., :K]
    return inp


def _expand(inp, H, N):
    """The same inputs with one B/C row per head (np.repeat over each group's
    heads) and theta zero-padded to all N/2 pairs."""
    G = inp["B"].shape[2]
    out = dict(inp)
    out["B"] = np.repeat(inp["B"], H // G, axis=2)
    out["C"] = np.repeat(inp["C"], H // G, axis=2)
    th = np.zeros(inp["theta"].shape[:-1] + (N // 2,))
    th[..., :inp["theta"].shape[-1]] = inp["theta"]
    out["theta"] = th
    return out


@pytest.mark.parametrize("G,K", [(1, 3), (2, 1), (6, 2), (3, 4)])
def test_grouped_partial_siso(oracle_mod, G, K):
    rng = np.random.default_rng(60 + 7 * G + K)
    Bt, T, H, P, N = 2, 9, 6, 3, 8
    inp = _grouped(rng, Bt, T, H, G, P, N, 1, K)
    full = _expand(inp, H, N)
    nrm = dict(normw_B=1 + 0.2 * rng.standard_normal(N), normw_C=1 + 0.2 * rng.standard_normal(N),
               bias_B=rng.standard_normal((H, 1, N)), bias_C=rng.standard_normal((H, 1, N)), eps=1e-5)
    a0 = rng.uniform(-2, 2, (Bt, H, K))
    a0f = np.zeros((Bt, H, N // 2))
    a0f[..., :K] = a0
    got = oracle_mod.siso_loop(**inp, angle0=a0, norm=nrm)
    ref = oracle_mod.siso_loop(**full, angle0=a0f, norm=nrm)
    for gg, rr in zip(got[:3], ref[:3]):
        close(gg, rr)
    close(got[3], ref[3][..., :K])
    close(ref[3][..., K:], 0.0)
    ch = oracle_mod.siso_chunked(**inp, chunk=4, angle0=a0, norm=nrm)
    for gg, rr in zip(ch, got):
        close(gg, rr, rtol=1e-9)


@pytest.mark.parametrize("G,K,R", [(2, 2, 2), (1, 3, 3)])
def test_grouped_partial_mimo_and_decode(oracle_mod, G, K, R):
    rng = np.random.default_rng(70 + G + K + R)
    Bt, T, H, P, N = 2, 6, 4, 3, 8
    inp = _grouped(rng, Bt, T, H, G, P, N, R, K)
    Wx = 1 + 0.3 * rng.standard_normal((H, R, P))
    Wy = 1 + 0.3 * rng.standard_normal((H, R, P))
    full = _expand(inp, H, N)
    got = oracle_mod.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    ref = oracle_mod.mimo_loop(**full, Wx=Wx, Wy=Wy)
    for gg, rr in zip(got[:3], ref[:3]):
        close(gg, rr)
    close(got[3], ref[3][..., :K])
    # decode steps, full state and factored, on the grouped partial inputs
    h, u, a = np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N, P)), np.zeros((Bt, H, K))
    hf, bp, xp, af = h.copy(), np.zeros((Bt, H, R, N)), np.zeros((Bt, H, P)), a.copy()
    for t in range(T):
        yt, h, u, a = oracle_mod.mimo_step_decode(*_tok(inp, t), h, u, a, Wx=Wx, Wy=Wy)
        close(yt, got[0][:, t])
        yf, hf, bp, xp, af = oracle_mod.step_decode_factored(*_tok(inp, t), hf, bp, xp, af, Wx=Wx, Wy=Wy)
        close(yf, got[0][:, t])
    close(h, got[1])
    close(u, got[2])
    close(hf, got[1])
    close(a, got[3])


def test_grouped_partial_siso_decode(oracle_mod):
    rng = np.random.default_rng(75)
    Bt, T, H, G, P, N, K = 2, 5, 4, 2, 3, 8, 2
    inp = _grouped(rng, Bt, T, H, G, P, N, 1, K)
    y1, h1, u1, a1 = oracle_mod.siso_loop(**inp)
    h, u, a = np.zeros((Bt, H, N, P)), np.zeros((Bt, H, N, P)), np.zeros((Bt, H, K))
    for t in range(T):
        yt, h, u, a = oracle_mod.step_decode(*_tok(inp, t), h, u, a)
        close(yt, y1[:, t])
    close(h, h1)
    close(u, u1)
    close(a, a1)


def test_partial_rope_turns_only_first_pairs(oracle_mod):
    rng = np.random.default_rng(76)
    Bt, T, H, G, N, K = 2, 7, 4, 2, 10, 3
    inp = _grouped(rng, Bt, T, H, G, 2, N, 1, K)
    Br, Cr, ang = oracle_mod.rope_bc(inp["B"], inp["C"], inp["theta"], inp["dt"])
    assert Br.shape == (Bt, T, H, N) and ang.shape == (Bt, H, K)
    Bh = np.repeat(inp["B"], H // G, axis=2)
    np.testing.assert_array_equal(Br[..., 2 * K:], Bh[..., 2 * K:])
    phi = np.cumsum(inp["dt"][..., None] * inp["theta"], axis=1)
    zb = (Bh[..., 0:2 * K:2] + 1j * Bh[..., 1:2 * K:2]) * np.exp(1j * phi)
    close(Br[..., 0:2 * K:2] + 1j * Br[..., 1:2 * K:2], zb)
    close(ang, phi[:, -1])


def test_bad_groups_and_pairs(oracle_mod):
    rng = np.random.default_rng(77)
    inp = _grouped(rng, 1, 3, 6, 4, 2, 8, 1, 2)     # 6 heads, 4 groups
    with pytest.raises(ValueError):
        oracle_mod.siso_loop(**inp)
    inp = _grouped(rng, 1, 3, 6, 3, 2, 8, 1, 4)
    inp["theta"] = np.zeros((1, 3, 6, 5))            # 5 pairs of 4 available
    with pytest.raises(ValueError):
        oracle_mod.siso_loop(**inp)


# ----------------------------------------------------------------------------
# chunked fp64 form (shifted-gamma fold) == loop
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("Q", [1, 4, 16, 64])
@pytest.mark.parametrize("T", [1, 5, 37])
def test_chunked_equals_loop(oracle_mod, Q, T):
    rng = np.random.default_rng(12 + Q + T)
    inp = rnd_inputs(rng, Bt=1, T=T, H=2, P=3, N=4)
    h0 = rng.standard_normal((1, 2, 4, 3))
    u0 = rng.standard_normal((1, 2, 4, 3))
    a0 = rng.uniform(-2, 2, (1, 2, 2))
    ref = oracle_mod.siso_loop(**inp, h0=h0, prevBx0=u0, angle0=a0)
    got = oracle_mod.siso_chunked(**inp, chunk=Q, h0=h0, prevBx0=u0, angle0=a0)
    for a, b in zip(ref, got):
        close(a, b, rtol=1e-9)


# ----------------------------------------------------------------------------
# invariants of the rotation, the norm and the discretization
# ----------------------------------------------------------------------------
def test_rotation_invariance(oracle_mod):
    rng = np.random.default_rng(13)
    inp = rnd_inputs(rng)
    y0, *_ = oracle_mod.siso_loop(**inp)
    shift = rng.uniform(-10, 10, (2, 3, 3))
    y1, *_ = oracle_mod.siso_loop(**inp, angle0=shift)
    close(y0, y1, rtol=1e-9)


def test_rope_zero_theta_is_identity_and_norm_preserving(oracle_mod):
    rng = np.random.default_rng(14)
    inp = rnd_inputs(rng)
    Br, Cr, ang = oracle_mod.rope_bc(inp["B"], inp["C"], np.zeros_like(inp["theta"]), inp["dt"])
    np.testing.assert_array_equal(Br, inp["B"])
    np.testing.assert_array_equal(Cr, inp["C"])
    Br, Cr, ang = oracle_mod.rope_bc(inp["B"], inp["C"], inp["theta"], inp["dt"])
    pn = lambda v: v[..., 0::2] ** 2 + v[..., 1::2] ** 2
    close(pn(Br), pn(inp["B"]))
    # as complex numbers the rotation is a multiplication by exp(i Phi_t)
    phi = np.cumsum(inp["dt"][..., None] * inp["theta"], axis=1)
    zb = (inp["B"][..., 0::2] + 1j * inp["B"][..., 1::2]) * np.exp(1j * phi)
    close(Br[..., 0::2] + 1j * Br[..., 1::2], zb)


def test_qknorm_and_bias(oracle_mod):
    rng = np.random.default_rng(15)
    inp = rnd_inputs(rng, N=8)
    H, N = 3, 8
    ones = np.ones(N)
    zero_theta = np.zeros_like(inp["theta"])
    nrm = dict(normw_B=ones, normw_C=ones, eps=0.0)
    Br, Cr, _ = oracle_mod.rope_bc(inp["B"], inp["C"], zero_theta, inp["dt"], norm=nrm)
    close(np.sqrt((Br ** 2).mean(-1)), np.ones(Br.shape[:-1]))
    Br3, _, _ = oracle_mod.rope_bc(3.0 * inp["B"], inp["C"], zero_theta, inp["dt"], norm=nrm)
    close(Br3, Br)
    bias = rng.standard_normal((H, 1, N))
    Bb, _, _ = oracle_mod.rope_bc(inp["B"], inp["C"], zero_theta, inp["dt"],
                                  norm=dict(bias_B=bias, eps=0.0))
    close(Bb, inp["B"] + bias[None, None, :, 0, :])


def test_trapezoid_weights(oracle_mod):
    rng = np.random.default_rng(16)
    inp = rnd_inputs(rng)
    al, be, ga = oracle_mod.discretize(inp["dt"], inp["A"], inp["lam"])
    close(be / al + ga, inp["dt"])         # the two trapezoid weights sum to dt
    lam0 = np.zeros_like(inp["lam"])
    al, be, ga = oracle_mod.discretize(inp["dt"], inp["A"], lam0)
    assert np.all(ga == 0.0)


def test_bad_arguments(oracle_mod):
    rng = np.random.default_rng(17)
    inp = rnd_inputs(rng, N=6)
    inp["B"] = inp["B"][..., :5]
    inp["C"] = inp["C"][..., :5]
    with pytest.raises(ValueError):
        oracle_mod.siso_loop(**inp)
