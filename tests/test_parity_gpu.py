"""GPU parity: every C-ABI entry point against the fp64 oracle on the same
seeded inputs (marked gpu).

Small cases compare every element and span several chunks with a ragged tail;
the full-size workloads compare whole sampled (b, h) lanes, which the oracle
computes exactly because lanes are independent.  Bars: max relative error
(normwise) 1e-5 for fp32 inputs, 2e-2 for bf16 inputs; final h and prev_Bx and
the angle are compared as well as y.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, Canary, cuda, lane_inputs, norm_dev, norm_f64, relerr, sample_lanes
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.inputs import to_f64

pytestmark = pytest.mark.gpu

FP32, BF16 = "f32", "bf16"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
    oracle.build_oracle()


def _tol(dtype):
    return TOL[gen.storage_dtype(dtype)]


def _states(Bt, H, N, P, seed):
    g = torch.Generator().manual_seed(seed)
    h0 = torch.randn(Bt, H, N, P, generator=g, dtype=torch.float64).float() * 0.5
    u0 = torch.randn(Bt, H, N, P, generator=g, dtype=torch.float64).float() * 0.1
    a0 = (torch.rand(Bt, H, N // 2, generator=g, dtype=torch.float64) * 6 - 3).float()
    return h0, u0, a0


# ----------------------------------------------------------------------------
# S1 discretize
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(2, 37, 3), (8, 2048, 16)])
def test_discretize(shape):
    Bt, T, H = shape
    inp = gen.scan_inputs(Bt, T, H, 4, 4, seed=11)
    d = cuda(inp)
    al, be, ga = m3.discretize(d["dt"], d["A"], d["lam"])
    ra, rb, rg = oracle.discretize(to_f64(inp["dt"]), to_f64(inp["A"]), to_f64(inp["lam"]))
    for got, ref in ((al, ra), (be, rb), (ga, rg)):
        assert relerr(got, ref) <= 1e-6


# ----------------------------------------------------------------------------
# S2 rope
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [FP32, BF16])
@pytest.mark.parametrize("R,T,N,bcnorm", [(1, 1, 4, False), (1, 77, 16, True), (3, 40, 8, True),
                                          (1, 300, 128, False), (4, 65, 128, True)])
def test_rope_bc(dtype, R, T, N, bcnorm):
    inp = gen.scan_inputs(2, T, 3, 4, N, rank=R, dtype=dtype, seed=12 + T, mimo_weights=R > 1,
                          bcnorm=bcnorm)
    _, _, a0 = _states(2, 3, N, 4, 5)
    d = cuda(inp)
    Br, Cr, ang = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"], angle0=a0.cuda(), norm=norm_dev(inp))
    rB, rC, rA = oracle.rope_bc(to_f64(inp["B"]), to_f64(inp["C"]), to_f64(inp["theta"]),
                                to_f64(inp["dt"]), angle0=to_f64(a0), norm=norm_f64(inp))
    tol = _tol(dtype)
    assert relerr(Br, rB) <= tol
    assert relerr(Cr, rC) <= tol
    assert relerr(ang, rA) <= 1e-5


@pytest.mark.parametrize("dtype", [FP32, BF16])
@pytest.mark.parametrize("N,R,bcnorm,T", [(128, 1, False, 700), (256, 1, True, 100), (256, 2, False, 65),
                                          (64, 1, True, 1), (128, 4, True, 33)])
def test_rope_bc_tiles(dtype, N, R, bcnorm, T):
    """The tiled rotation (whole quads of pairs): several tiles with a ragged
    last one, the angle carried from tile to tile, a slice of a row per CTA
    without QkNorm and the whole row with it (dstate 256: one token per warp)."""
    inp = gen.scan_inputs(2, T, 3, 4, N, rank=R, dtype=dtype, seed=13 + N + T, mimo_weights=R > 1,
                          bcnorm=bcnorm)
    _, _, a0 = _states(2, 3, N, 4, 6)
    d = cuda(inp)
    Br, Cr, ang = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"], angle0=a0.cuda(), norm=norm_dev(inp))
    rB, rC, rA = oracle.rope_bc(to_f64(inp["B"]), to_f64(inp["C"]), to_f64(inp["theta"]),
                                to_f64(inp["dt"]), angle0=to_f64(a0), norm=norm_f64(inp))
    tol = _tol(dtype)
    assert relerr(Br, rB) <= tol
    assert relerr(Cr, rC) <= tol
    assert relerr(ang, rA) <= 1e-5


def test_rope_bc_empty_sequence_passes_the_angle_through():
    inp = gen.scan_inputs(2, 0, 3, 4, 128, seed=14)
    _, _, a0 = _states(2, 3, 128, 4, 8)
    d = cuda(inp)
    _, _, ang = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"], angle0=a0.cuda())
    torch.cuda.synchronize()
    assert torch.equal(ang.cpu(), a0)


def test_rope_bc_full_size_sampled_lanes():
    """The standalone rotation at the default workload's shape (the S2 bench
    line), compared on sampled (b, h) lanes."""
    inp = gen.config_inputs(1)
    d = cuda({k: inp[k] for k in ("B", "C", "theta", "dt")})
    Br, Cr, ang = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"])
    torch.cuda.synchronize()
    for b, h in sample_lanes(8, 16):
        sl = lambda t: to_f64(t[b:b + 1, :, h:h + 1])
        rB, rC, rA = oracle.rope_bc(sl(inp["B"]), sl(inp["C"]), sl(inp["theta"]), sl(inp["dt"]))
        assert relerr(Br[b:b + 1, :, h:h + 1], rB) <= 2e-2
        assert relerr(Cr[b:b + 1, :, h:h + 1], rC) <= 2e-2
        assert relerr(ang[b:b + 1, h:h + 1], rA) <= 1e-5


# ----------------------------------------------------------------------------
# S3 SISO chunked scan: small cases, every element
# ----------------------------------------------------------------------------
def _siso_check(inp, chunk, with_state=False, seed=0):
    Bt, T, H, P = inp["x"].shape
    N = inp["B"].shape[-1]
    h0 = u0 = a0 = None
    if with_state:
        h0, u0, a0 = _states(Bt, H, N, P, seed)
    d = cuda(inp)
    ycan = Canary((Bt, T, H, P), inp["x"].dtype)
    hcan = Canary((Bt, H, N, P), torch.float32)
    out = (ycan.t, hcan.t, torch.empty(Bt, H, N, P, device="cuda"), torch.empty(Bt, H, N // 2, device="cuda"))
    y, hf, uf, af = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                                        d["D"], chunk, norm=norm_dev(inp),
                                        h0=None if h0 is None else h0.cuda(),
                                        prevBx0=None if u0 is None else u0.cuda(),
                                        angle0=None if a0 is None else a0.cuda(), out=out)
    torch.cuda.synchronize()
    ycan.check()
    hcan.check()
    ref = oracle.siso_loop(**{k: to_f64(inp[k]) for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")},
                           h0=None if h0 is None else to_f64(h0),
                           prevBx0=None if u0 is None else to_f64(u0),
                           angle0=None if a0 is None else to_f64(a0), norm=norm_f64(inp))
    return [relerr(g, r) for g, r in zip((y, hf, uf, af), ref)]


def test_config0_tiny_fp32():
    c = gen.CONFIGS[0]
    inp = gen.config_inputs(0)
    errs = _siso_check(inp, c["chunk"])
    assert max(errs) <= 1e-5, errs


@pytest.mark.parametrize("T", [1, 3, 15, 16, 17, 64, 100])
@pytest.mark.parametrize("chunk", [16, 7])
def test_siso_fp32_edges(T, chunk):
    inp = gen.scan_inputs(2, T, 3, 8, 6, dtype=FP32, seed=100 + T + chunk)
    errs = _siso_check(inp, chunk, with_state=True, seed=T)
    assert max(errs) <= 1e-5, errs


def test_siso_fp32_norm_bias():
    inp = gen.scan_inputs(2, 50, 2, 8, 16, dtype=FP32, seed=31, bcnorm=True)
    errs = _siso_check(inp, 16, with_state=True, seed=3)
    assert max(errs) <= 1e-5, errs


@pytest.mark.parametrize("T,chunk", [(150, 64), (64, 64), (1, 64), (300, 128)])
def test_siso_bf16_layer_shape(T, chunk):
    inp = gen.scan_inputs(2, T, 3, 64, 128, dtype=BF16, seed=40 + T)
    errs = _siso_check(inp, chunk, with_state=True, seed=T)
    assert max(errs) <= 2e-2, errs


@pytest.mark.parametrize("dt_shift,T", [(3.0, 200), (1.0, 130), (-6.0, 256)])
def test_siso_bf16_decay_regimes(dt_shift, T):
    # dt_shift 3: every chunk's log-decay range exceeds 60 (exact-mask path);
    # 1: a mix; -6: almost no decay (long memory)
    inp = gen.scan_inputs(2, T, 2, 64, 128, dtype=BF16, dt_shift=dt_shift, seed=int(50 + T))
    errs = _siso_check(inp, 64, with_state=True, seed=T)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


def test_siso_bf16_norm_bias():
    inp = gen.scan_inputs(1, 130, 2, 64, 128, dtype=BF16, seed=41, bcnorm=True)
    errs = _siso_check(inp, 64)
    assert max(errs) <= 2e-2, errs


@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 63, 64, 65, 127, 129, 1000])
def test_siso_bf16_ragged_lengths(T):
    inp = gen.scan_inputs(3, T, 2, 64, 128, dtype=BF16, seed=90 + T)
    errs = _siso_check(inp, 64, with_state=(T % 2 == 1), seed=T)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


@pytest.mark.parametrize("Bt,H,T,with_state", [(1, 2, 3000, True), (1, 1, 1000, False), (2, 3, 2560, True),
                                                (1, 2, 600, True)])
def test_siso_bf16_segmented_long_sequences(Bt, H, T, with_state):
    # few lanes and long sequences: each lane is cut into segments that run in
    # parallel (state-only pass, combine pass, full pass with workspace)
    d = m3.Dims(Bt, T, H, 64, 128, 1, 64)
    assert m3.workspace_bytes(m3.M3_WS_SISO, d, m3.M3_BF16) > 0
    inp = gen.scan_inputs(Bt, T, H, 64, 128, dtype=BF16, seed=300 + T, dt_shift=-4.0)
    errs = _siso_check(inp, 64, with_state=with_state, seed=T)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


def test_siso_empty_sequence_passes_state_through():
    inp = gen.scan_inputs(2, 0, 3, 8, 6, dtype=FP32, seed=5)
    h0, u0, a0 = _states(2, 3, 6, 8, 9)
    d = cuda(inp)
    y, hf, uf, af = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                                        d["D"], 16, h0=h0.cuda(), prevBx0=u0.cuda(), angle0=a0.cuda())
    assert torch.equal(hf.cpu(), h0) and torch.equal(uf.cpu(), u0) and torch.equal(af.cpu(), a0)


@pytest.mark.parametrize("case", ["siso", "mimo_r4", "siso_segmented"])
def test_tc_scan_deterministic(case):
    """The scans use no atomics on the data path: two calls on the same
    inputs agree bit for bit (a race between warps or CTAs would show here)."""
    if case == "mimo_r4":
        inp = gen.scan_inputs(2, 200, 4, 64, 128, rank=4, dtype=BF16, seed=8)
    elif case == "siso_segmented":
        inp = gen.scan_inputs(1, 3000, 2, 64, 128, dtype=BF16, seed=9, dt_shift=-4.0)
    else:
        inp = gen.scan_inputs(2, 200, 4, 64, 128, dtype=BF16, seed=7)
    d = cuda(inp)

    def run():
        if case == "mimo_r4":
            return m3.mimo_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"], 64,
                                       W_x=d["Wx"], W_y=d["Wy"])
        return m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"], 64)

    a, b = run(), run()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


# ----------------------------------------------------------------------------
# S4 MIMO
# ----------------------------------------------------------------------------
def _mimo_check(inp, chunk, with_state=False, seed=0):
    Bt, T, H, P = inp["x"].shape
    N = inp["B"].shape[-1]
    h0 = u0 = a0 = None
    if with_state:
        h0, u0, a0 = _states(Bt, H, N, P, seed)
    d = cuda(inp)
    y, hf, uf, af = m3.mimo_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                                        d["D"], chunk, W_x=d.get("Wx"), W_y=d.get("Wy"), norm=norm_dev(inp),
                                        h0=None if h0 is None else h0.cuda(),
                                        prevBx0=None if u0 is None else u0.cuda(),
                                        angle0=None if a0 is None else a0.cuda())
    ref = oracle.mimo_loop(**{k: to_f64(inp[k]) for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")},
                           Wx=to_f64(inp["Wx"]), Wy=to_f64(inp["Wy"]),
                           h0=None if h0 is None else to_f64(h0),
                           prevBx0=None if u0 is None else to_f64(u0),
                           angle0=None if a0 is None else to_f64(a0), norm=norm_f64(inp))
    return [relerr(g, r) for g, r in zip((y, hf, uf, af), ref)]


@pytest.mark.parametrize("R,T,chunk", [(1, 20, 8), (2, 33, 8), (4, 17, 16), (3, 1, 4)])
def test_mimo_fp32(R, T, chunk):
    inp = gen.scan_inputs(2, T, 2, 8, 8, rank=R, dtype=FP32, seed=60 + R + T, mimo_weights=True)
    errs = _mimo_check(inp, chunk, with_state=True, seed=R)
    assert max(errs) <= 1e-5, errs


def test_mimo_fp32_norm_bias():
    inp = gen.scan_inputs(1, 30, 2, 8, 8, rank=2, dtype=FP32, seed=61, mimo_weights=True, bcnorm=True)
    errs = _mimo_check(inp, 8)
    assert max(errs) <= 1e-5, errs


@pytest.mark.parametrize("R,T", [(4, 40), (4, 129), (4, 1), (4, 17), (2, 100), (2, 33)])
def test_mimo_bf16_layer_shape(R, T):
    # headdim 64, dState 128, rank 2 or 4: the tensor-core path (64 rows per chunk)
    inp = gen.scan_inputs(2, T, 2, 64, 128, rank=R, dtype=BF16, seed=62 + T + R, mimo_weights=True)
    errs = _mimo_check(inp, 64, with_state=True, seed=4)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


def test_mimo_bf16_norm_bias():
    inp = gen.scan_inputs(1, 70, 2, 64, 128, rank=4, dtype=BF16, seed=65, mimo_weights=True, bcnorm=True)
    errs = _mimo_check(inp, 64, with_state=True, seed=5)
    assert max(errs) <= 2e-2, errs


@pytest.mark.parametrize("R,T", [(4, 1000), (2, 700)])
def test_mimo_bf16_segmented(R, T):
    d = m3.Dims(1, T, 2, 64, 128, R, 64)
    assert m3.workspace_bytes(m3.M3_WS_MIMO, d, m3.M3_BF16) > 0
    inp = gen.scan_inputs(1, T, 2, 64, 128, rank=R, dtype=BF16, seed=66 + T, mimo_weights=True, dt_shift=-4.0)
    errs = _mimo_check(inp, 64, with_state=True, seed=6)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


# ----------------------------------------------------------------------------
# S5 decode
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,P,N", [(FP32, 8, 6), (FP32, 5, 4), (BF16, 64, 128)])
def test_decode_steps(dtype, P, N):
    Bt, H, T0, steps = 3, 2, 9, 8
    inp = gen.scan_inputs(Bt, T0, H, P, N, dtype=dtype, seed=70 + P)
    d = cuda(inp)
    _, h, u, a = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"], 4)
    ref = oracle.siso_loop(**{k: to_f64(inp[k]) for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")})
    rh, ru, ra = ref[1], ref[2], ref[3]
    g = inp["generator"]
    tol = _tol(dtype)
    for s in range(steps):
        st = gen.decode_step_inputs(g, Bt, H, P, N, dtype=dtype)
        ds = cuda(st)
        y = m3.step_decode(ds["x"], ds["dt"], d["A"], ds["lam"], ds["theta"], ds["B"], ds["C"], d["D"], h, u, a)
        ry, rh, ru, ra = oracle.step_decode(to_f64(st["x"]), to_f64(st["dt"]), to_f64(inp["A"]),
                                            to_f64(st["lam"]), to_f64(st["theta"]), to_f64(st["B"]),
                                            to_f64(st["C"]), to_f64(inp["D"]), rh, ru, ra)
        assert relerr(y, ry) <= tol
    assert relerr(h, rh) <= tol and relerr(u, ru) <= tol and relerr(a, ra) <= 1e-5


def test_decode_norm_bias():
    Bt, H, P, N = 2, 2, 8, 8
    inp = gen.scan_inputs(Bt, 1, H, P, N, dtype=FP32, seed=80, bcnorm=True)
    h0, u0, a0 = _states(Bt, H, N, P, 1)
    d = cuda(inp)
    h, u, a = h0.cuda(), u0.cuda(), a0.cuda()
    y = m3.step_decode(d["x"][:, 0].contiguous(), d["dt"][:, 0].contiguous(), d["A"],
                       d["lam"][:, 0].contiguous(), d["theta"][:, 0].contiguous(), d["B"][:, 0].contiguous(),
                       d["C"][:, 0].contiguous(), d["D"], h, u, a, norm=norm_dev(inp))
    nf = norm_f64(inp)
    nf["bias_B"] = nf["bias_B"][:, 0]
    nf["bias_C"] = nf["bias_C"][:, 0]
    ry, rh, ru, ra = oracle.step_decode(to_f64(inp["x"][:, 0]), to_f64(inp["dt"][:, 0]), to_f64(inp["A"]),
                                        to_f64(inp["lam"][:, 0]), to_f64(inp["theta"][:, 0]),
                                        to_f64(inp["B"][:, 0]), to_f64(inp["C"][:, 0]), to_f64(inp["D"]),
                                        to_f64(h0), to_f64(u0), to_f64(a0), norm=nf)
    for g, r in ((y, ry), (h, rh), (u, ru), (a, ra)):
        assert relerr(g, r) <= 1e-5


# ----------------------------------------------------------------------------
# S5 for rank R, and decode on the factored previous-input state
# ----------------------------------------------------------------------------
def _mimo_w(g, H, R, P):
    w = lambda: (1.0 + 0.3 * torch.randn(H, R, P, generator=g, dtype=torch.float64)).float()
    return w(), w()


def _dec_step(st, d, R):
    """Per-token device inputs (B, C with the rank axis) of one decode step."""
    ds = cuda(st)
    return (ds["x"], ds["dt"], d["A"], ds["lam"], ds["theta"], ds["B"], ds["C"], d["D"])


def _dec_step_f64(st, inp):
    return (to_f64(st["x"]), to_f64(st["dt"]), to_f64(inp["A"]), to_f64(st["lam"]), to_f64(st["theta"]),
            to_f64(st["B"]), to_f64(st["C"]), to_f64(inp["D"]))


@pytest.mark.parametrize("dtype", [FP32, BF16])
@pytest.mark.parametrize("R", [2, 4])
def test_mimo_decode_steps(dtype, R):
    Bt, H, P, N, steps = 3, 2, 16, 8, 6
    inp = gen.scan_inputs(Bt, 1, H, P, N, rank=R, dtype=dtype, seed=90 + R)
    d = cuda(inp)
    g = torch.Generator().manual_seed(190 + R)
    Wx, Wy = _mimo_w(g, H, R, P)
    h0, u0, a0 = _states(Bt, H, N, P, 91 + R)
    h, u, a = h0.cuda(), u0.cuda(), a0.cuda()
    rh, ru, ra = to_f64(h0), to_f64(u0), to_f64(a0)
    tol = _tol(dtype)
    for _ in range(steps):
        st = gen.decode_step_inputs(g, Bt, H, P, N, dtype=dtype, rank=R)
        y = m3.mimo_step_decode(*_dec_step(st, d, R), h, u, a, W_x=Wx.cuda(), W_y=Wy.cuda())
        ry, rh, ru, ra = oracle.mimo_step_decode(*_dec_step_f64(st, inp), rh, ru, ra, Wx=to_f64(Wx),
                                                 Wy=to_f64(Wy))
        assert relerr(y, ry) <= tol
    assert relerr(h, rh) <= tol and relerr(u, ru) <= tol and relerr(a, ra) <= 1e-5


@pytest.mark.parametrize("dtype", [FP32, BF16])
@pytest.mark.parametrize("R", [1, 3, 4])
def test_factored_decode_steps(dtype, R):
    Bt, H, P, N, steps = 3, 2, 16, 8, 6
    inp = gen.scan_inputs(Bt, 1, H, P, N, rank=max(R, 2), dtype=dtype, seed=95 + R)
    d = cuda(inp)
    g = torch.Generator().manual_seed(195 + R)
    Wx, Wy = _mimo_w(g, H, R, P)
    h0, _, a0 = _states(Bt, H, N, P, 96 + R)
    bp0 = (torch.randn(Bt, H, R, N, generator=g, dtype=torch.float64) / N ** 0.5).float()
    xp0 = torch.randn(Bt, H, P, generator=g, dtype=torch.float64).float()
    h, bp, xp, a = h0.cuda(), bp0.cuda(), xp0.cuda(), a0.cuda()
    rh, rbp, rxp, ra = to_f64(h0), to_f64(bp0), to_f64(xp0), to_f64(a0)
    tol = _tol(dtype)
    for _ in range(steps):
        st = gen.decode_step_inputs(g, Bt, H, P, N, dtype=dtype, rank=R, rank_axis=True)
        y = m3.step_decode_factored(*_dec_step(st, d, R), h, bp, xp, a, W_x=Wx.cuda(), W_y=Wy.cuda())
        ry, rh, rbp, rxp, ra = oracle.step_decode_factored(*_dec_step_f64(st, inp), rh, rbp, rxp, ra,
                                                           Wx=to_f64(Wx), Wy=to_f64(Wy))
        assert relerr(y, ry) <= tol
    assert relerr(h, rh) <= tol and relerr(bp, rbp) <= tol and relerr(a, ra) <= 1e-5
    assert relerr(xp, rxp) == 0.0          # x_prev is x_t itself


def test_factored_decode_norm_bias():
    Bt, H, P, N, R = 2, 2, 8, 8, 2
    inp = gen.scan_inputs(Bt, 1, H, P, N, rank=R, dtype=FP32, seed=98, bcnorm=True)
    g = torch.Generator().manual_seed(198)
    Wx, Wy = _mimo_w(g, H, R, P)
    h0, _, a0 = _states(Bt, H, N, P, 99)
    bp0 = torch.randn(Bt, H, R, N, generator=g, dtype=torch.float64).float()
    xp0 = torch.randn(Bt, H, P, generator=g, dtype=torch.float64).float()
    d = cuda(inp)
    h, bp, xp, a = h0.cuda(), bp0.cuda(), xp0.cuda(), a0.cuda()
    tok = lambda k: d[k][:, 0].contiguous()
    y = m3.step_decode_factored(tok("x"), tok("dt"), d["A"], tok("lam"), tok("theta"), tok("B"), tok("C"), d["D"],
                                h, bp, xp, a, W_x=Wx.cuda(), W_y=Wy.cuda(), norm=norm_dev(inp))
    f = lambda k: to_f64(inp[k][:, 0])
    ry, rh, rbp, rxp, ra = oracle.step_decode_factored(f("x"), f("dt"), to_f64(inp["A"]), f("lam"), f("theta"),
                                                       f("B"), f("C"), to_f64(inp["D"]), to_f64(h0), to_f64(bp0),
                                                       to_f64(xp0), to_f64(a0), Wx=to_f64(Wx), Wy=to_f64(Wy),
                                                       norm=norm_f64(inp))
    for got, ref in ((y, ry), (h, rh), (bp, rbp), (a, ra)):
        assert relerr(got, ref) <= 1e-5


@pytest.mark.parametrize("R", [1, 2])
def test_prefill_then_factored_decode(R):
    """A chunked prefill on the GPU, its last token's rotated B (m3_rope_bc)
    and x as the factored state, then decode steps: equal to the one-shot
    oracle scan over prefill + decoded tokens."""
    Bt, H, P, N, T0, steps = 2, 3, 16, 8, 11, 5
    T = T0 + steps
    full = gen.scan_inputs(Bt, T, H, P, N, rank=R, dtype=FP32, seed=101 + R, mimo_weights=True)
    pre = {k: (v[:, :T0].contiguous() if k in ("x", "dt", "lam", "theta", "B", "C") else v)
           for k, v in full.items() if isinstance(v, torch.Tensor)}
    d = cuda(pre)
    _, h, _, a = m3.mimo_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"], 4,
                                     W_x=d["Wx"], W_y=d["Wy"])
    Br, _, _ = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"])
    bp = Br[:, T0 - 1].float().contiguous()
    xp = d["x"][:, T0 - 1].float().contiguous()
    ys = []
    fd = cuda(full)
    for t in range(T0, T):
        tk = lambda k: fd[k][:, t].contiguous()
        ys.append(m3.step_decode_factored(tk("x"), tk("dt"), fd["A"], tk("lam"), tk("theta"), tk("B"), tk("C"),
                                          fd["D"], h, bp, xp, a, W_x=fd["Wx"], W_y=fd["Wy"]))
    ref = oracle.mimo_loop(**{k: to_f64(full[k]) for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")},
                           Wx=to_f64(full["Wx"]), Wy=to_f64(full["Wy"]))
    assert relerr(torch.stack(ys, 1), ref[0][:, T0:]) <= 1e-5
    assert relerr(h, ref[1]) <= 1e-5 and relerr(a, ref[3]) <= 1e-5


# ----------------------------------------------------------------------------
# full-size workloads, sampled lanes (the launch configuration the bench times)
# ----------------------------------------------------------------------------
def _full_scan(idx):
    c = gen.CONFIGS[idx]
    inp = gen.config_inputs(idx)
    d = cuda(inp)
    if c["rank"] > 1:
        out = m3.mimo_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"],
                                  c["chunk"], W_x=d["Wx"], W_y=d["Wy"])
    else:
        out = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"],
                                  c["chunk"])
    torch.cuda.synchronize()
    y, hf, uf, af = (t.cpu() for t in out)
    for (b, h) in sample_lanes(c["batch"], c["nheads"]):
        li = lane_inputs(inp, b, h)
        if c["rank"] > 1:
            ref = oracle.mimo_loop(**li)
        else:
            ref = oracle.siso_loop(**li)
        got = (y[b:b + 1, :, h:h + 1], hf[b:b + 1, h:h + 1], uf[b:b + 1, h:h + 1], af[b:b + 1, h:h + 1])
        errs = [relerr(g, r) for g, r in zip(got, ref)]
        assert max(errs) <= 2e-2, (idx, b, h, errs)
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("idx", [1, 2, 3])
def test_full_size_sampled_lanes(idx):
    _full_scan(idx)


def test_full_size_decode_sampled_lanes():
    c = gen.CONFIGS[4]
    Bt, H, P, N = c["batch"], c["nheads"], c["headdim"], c["dstate"]
    inp = gen.config_inputs(4)
    d = cuda(inp)
    _, h, u, a = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"],
                                     c["chunk"])
    lanes = sample_lanes(Bt, H)
    g = inp["generator"]
    seq = {k: [] for k in ("x", "dt", "lam", "theta", "B", "C")}
    ys = []
    for s in range(c["steps"]):
        st = gen.decode_step_inputs(g, Bt, H, P, N)
        ds = cuda(st)
        y = m3.step_decode(ds["x"], ds["dt"], d["A"], ds["lam"], ds["theta"], ds["B"], ds["C"], d["D"], h, u, a)
        ys.append(torch.stack([y[b, hh] for (b, hh) in lanes]).cpu())
        for k in seq:
            seq[k].append(torch.stack([st[k][b, hh] for (b, hh) in lanes]))
    torch.cuda.synchronize()
    ys = torch.stack(ys, 1)                         # (lanes, steps, P)
    for li_, (b, hh) in enumerate(lanes):
        li = lane_inputs(inp, b, hh)
        # the prefill followed by the steps is one longer sequence for the oracle
        for k in ("x", "theta", "B", "C"):
            steps = torch.stack([v[li_] for v in seq[k]])[None, :, None]
            li[k] = np.concatenate([li[k], to_f64(steps)], axis=1)
        for k in ("dt", "lam"):
            steps = torch.stack([v[li_] for v in seq[k]])[None, :, None]
            li[k] = np.concatenate([li[k], to_f64(steps)], axis=1)
        ry, rh, ru, ra = oracle.siso_loop(**li)
        T0 = c["seqlen"]
        assert relerr(ys[li_], ry[0, T0:, 0]) <= 2e-2
        assert relerr(h[b, hh], rh[0, 0]) <= 2e-2
        assert relerr(u[b, hh], ru[0, 0]) <= 2e-2
        assert relerr(a[b, hh], ra[0, 0]) <= 1e-5


def test_full_size_factored_decode_sampled_lanes():
    """Decode workload shape, factored state: prefill, b_prev from the prefill's
    last rotated B (m3_rope_bc), then 64 steps; sampled lanes against the
    oracle's one-shot loop over prefill + steps."""
    c = gen.CONFIGS[4]
    Bt, H, P, N = c["batch"], c["nheads"], c["headdim"], c["dstate"]
    inp = gen.config_inputs(4)
    d = cuda(inp)
    T0 = c["seqlen"]
    _, h, _, a = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"],
                                     c["chunk"])
    Br, _, _ = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"])
    bp = Br[:, T0 - 1, :, None].float().contiguous()          # (Bt, H, 1, N)
    xp = d["x"][:, T0 - 1].float().contiguous()
    lanes = sample_lanes(Bt, H)
    g = inp["generator"]
    seq = {k: [] for k in ("x", "dt", "lam", "theta", "B", "C")}
    ys = []
    for s in range(64):
        st = gen.decode_step_inputs(g, Bt, H, P, N, rank_axis=True)
        ds = cuda(st)
        y = m3.step_decode_factored(ds["x"], ds["dt"], d["A"], ds["lam"], ds["theta"], ds["B"], ds["C"], d["D"],
                                    h, bp, xp, a)
        ys.append(torch.stack([y[b, hh] for (b, hh) in lanes]).cpu())
        for k in seq:
            v = st[k][:, :, 0] if k in ("B", "C") else st[k]
            seq[k].append(torch.stack([v[b, hh] for (b, hh) in lanes]))
    torch.cuda.synchronize()
    ys = torch.stack(ys, 1)
    for li_, (b, hh) in enumerate(lanes):
        li = lane_inputs(inp, b, hh)
        for k in seq:
            steps = torch.stack([v[li_] for v in seq[k]])[None, :, None]
            li[k] = np.concatenate([li[k], to_f64(steps)], axis=1)
        ry, rh, _, ra = oracle.siso_loop(**li)
        assert relerr(ys[li_], ry[0, T0:, 0]) <= 2e-2
        assert relerr(h[b, hh], rh[0, 0]) <= 2e-2
        assert relerr(a[b, hh], ra[0, 0]) <= 1e-5
