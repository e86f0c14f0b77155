"""GPU parity at the corners of the sizes the C ABI accepts (m3_get_limits):
dstate 256, headdim 256, dstate * headdim = 16384 and rank 8, for every
entry point that takes them -- the chunked forwards (the FFMA scan with its
largest shared-memory plans), the three decode steps (rank 8 at dstate 256
needs more than the default 48 KB of dynamic shared memory) and the backward
at its largest plans (chunk cut to fit 220 KB).  Each case is compared with
the fp64 oracle on the same stored inputs, every element, including the
final states and the angle (marked gpu)."""
import pytest
import torch

import oracle
from helpers import TOL, cuda, relerr
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.inputs import to_f64

pytestmark = pytest.mark.gpu

SCAN = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
BWD_TOL = 1e-4
NAME = {"dW_x": "dWx", "dW_y": "dWy"}


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
    oracle.build_oracle()


def test_limits_are_the_ones_covered_here():
    lim = m3.lib().m3_get_limits()
    assert (lim.max_dstate, lim.max_headdim, lim.max_state_elems, lim.max_rank) == (256, 256, 16384, 8)


def _seeded(shape, seed, scale):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * scale).float()


def _mimo_w(seed, H, R, P):
    return _seeded((H, R, P), seed, 0.3) + 1.0, _seeded((H, R, P), seed + 1, 0.3) + 1.0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,P,R", [(256, 64, 1), (64, 256, 1), (128, 128, 8), (256, 64, 8), (2, 256, 8)])
def test_chunked_fwd_at_the_size_limits(dtype, N, P, R):
    Bt, T, H = 1, 45, 2
    inp = gen.scan_inputs(Bt, T, H, P, N, rank=R, dtype=dtype, seed=900 + N + P + R)
    h0 = _seeded((Bt, H, N, P), 901, 0.5)
    u0 = _seeded((Bt, H, N, P), 902, 0.1)
    a0 = _seeded((Bt, H, N // 2), 903, 2.0)
    d = cuda(inp)
    args = [d[k] for k in SCAN]
    st = dict(h0=h0.cuda(), prevBx0=u0.cuda(), angle0=a0.cuda())
    ref_args = {k: to_f64(inp[k]) for k in SCAN}
    ref_st = dict(h0=to_f64(h0), prevBx0=to_f64(u0), angle0=to_f64(a0))
    if R == 1:
        got = m3.siso_chunked_fwd(*args, 64, **st)
        ref = oracle.siso_loop(**ref_args, **ref_st)
    else:
        Wx, Wy = _mimo_w(904, H, R, P)
        got = m3.mimo_chunked_fwd(*args, 64, W_x=Wx.cuda(), W_y=Wy.cuda(), **st)
        ref = oracle.mimo_loop(**ref_args, Wx=to_f64(Wx), Wy=to_f64(Wy), **ref_st)
    torch.cuda.synchronize()
    tol = TOL[gen.storage_dtype(dtype)]
    for g_, r_ in zip(got[:3], ref[:3]):
        assert relerr(g_, r_) <= tol
    assert relerr(got[3], ref[3]) <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,P", [(256, 64), (64, 256)])
def test_siso_decode_at_the_size_limits(dtype, N, P):
    Bt, H, steps = 2, 2, 3
    inp = gen.scan_inputs(Bt, 1, H, P, N, dtype=dtype, seed=910 + N)
    h0 = _seeded((Bt, H, N, P), 911, 0.5)
    u0 = _seeded((Bt, H, N, P), 912, 0.1)
    a0 = _seeded((Bt, H, N // 2), 913, 2.0)
    h, u, a = h0.cuda(), u0.cuda(), a0.cuda()
    rh, ru, ra = to_f64(h0), to_f64(u0), to_f64(a0)
    g = torch.Generator().manual_seed(914)
    tol = TOL[gen.storage_dtype(dtype)]
    for _ in range(steps):
        st = gen.decode_step_inputs(g, Bt, H, P, N, dtype=dtype)
        ds = cuda(st)
        y = m3.step_decode(ds["x"], ds["dt"], inp["A"].cuda(), ds["lam"], ds["theta"], ds["B"], ds["C"],
                           inp["D"].cuda(), h, u, a)
        ry, rh, ru, ra = oracle.step_decode(to_f64(st["x"]), to_f64(st["dt"]), to_f64(inp["A"]),
                                            to_f64(st["lam"]), to_f64(st["theta"]), to_f64(st["B"]),
                                            to_f64(st["C"]), to_f64(inp["D"]), rh, ru, ra)
        assert relerr(y, ry) <= tol
    assert relerr(h, rh) <= tol and relerr(u, ru) <= tol and relerr(a, ra) <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("factored", [False, True])
@pytest.mark.parametrize("N,P", [(256, 64), (128, 128), (64, 256)])
def test_rank8_decode_at_the_size_limits(dtype, factored, N, P):
    Bt, H, R, steps = 2, 2, 8, 3
    inp = gen.scan_inputs(Bt, 1, H, P, N, rank=R, dtype=dtype, seed=920 + N)
    Wx, Wy = _mimo_w(921, H, R, P)
    h0 = _seeded((Bt, H, N, P), 922, 0.5)
    a0 = _seeded((Bt, H, N // 2), 923, 2.0)
    h, a = h0.cuda(), a0.cuda()
    rh, ra = to_f64(h0), to_f64(a0)
    if factored:
        bp0 = _seeded((Bt, H, R, N), 924, N ** -0.5)
        xp0 = _seeded((Bt, H, P), 925, 1.0)
        bp, xp = bp0.cuda(), xp0.cuda()
        rbp, rxp = to_f64(bp0), to_f64(xp0)
    else:
        u0 = _seeded((Bt, H, N, P), 926, 0.1)
        u, ru = u0.cuda(), to_f64(u0)
    g = torch.Generator().manual_seed(927)
    tol = TOL[gen.storage_dtype(dtype)]
    for _ in range(steps):
        st = gen.decode_step_inputs(g, Bt, H, P, N, dtype=dtype, rank=R, rank_axis=True)
        ds = cuda(st)
        dev = (ds["x"], ds["dt"], inp["A"].cuda(), ds["lam"], ds["theta"], ds["B"], ds["C"], inp["D"].cuda())
        ref_in = (to_f64(st["x"]), to_f64(st["dt"]), to_f64(inp["A"]), to_f64(st["lam"]), to_f64(st["theta"]),
                  to_f64(st["B"]), to_f64(st["C"]), to_f64(inp["D"]))
        if factored:
            y = m3.step_decode_factored(*dev, h, bp, xp, a, W_x=Wx.cuda(), W_y=Wy.cuda())
            ry, rh, rbp, rxp, ra = oracle.step_decode_factored(*ref_in, rh, rbp, rxp, ra, Wx=to_f64(Wx),
                                                               Wy=to_f64(Wy))
        else:
            y = m3.mimo_step_decode(*dev, h, u, a, W_x=Wx.cuda(), W_y=Wy.cuda())
            ry, rh, ru, ra = oracle.mimo_step_decode(*ref_in, rh, ru, ra, Wx=to_f64(Wx), Wy=to_f64(Wy))
        assert relerr(y, ry) <= tol
    assert relerr(h, rh) <= tol and relerr(a, ra) <= 1e-5
    if factored:
        assert relerr(bp, rbp) <= tol and relerr(xp, rxp) == 0.0
    else:
        assert relerr(u, ru) <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,P,R", [(256, 64, 1), (64, 256, 1), (128, 64, 8), (128, 128, 8)])
def test_backward_at_its_largest_plans(dtype, N, P, R):
    Bt, T, H = 1, 21, 2
    inp = gen.scan_inputs(Bt, T, H, P, N, rank=R, dtype=dtype, seed=930 + N + P + R, mimo_weights=R > 1)
    h0 = _seeded((Bt, H, N, P), 931, 0.5)
    u0 = _seeded((Bt, H, N, P), 932, 0.2)
    a0 = _seeded((Bt, H, N // 2), 933, 2.0)
    dy = _seeded((Bt, T, H, P), 934, 1.0).to(inp["x"].dtype)
    adj = dict(dh_final=_seeded((Bt, H, N, P), 935, 0.3), dprevBx_final=_seeded((Bt, H, N, P), 936, 0.3),
               dangle_final=_seeded((Bt, H, N // 2), 937, 0.3))
    d = cuda(inp)
    kw = dict(h0=h0.cuda(), prevBx0=u0.cuda(), angle0=a0.cuda(), **{k: v.cuda() for k, v in adj.items()})
    if R > 1:
        kw["W_x"], kw["W_y"] = d["Wx"], d["Wy"]
    got = m3.chunked_bwd(*[d[k] for k in SCAN], dy.cuda(), 64, want=m3.GRAD_FIELDS, **kw)
    torch.cuda.synchronize()
    ref = oracle.loop_bwd(**{k: to_f64(inp[k]) for k in SCAN}, dy=to_f64(dy),
                          Wx=to_f64(inp["Wx"]) if R > 1 else None, Wy=to_f64(inp["Wy"]) if R > 1 else None,
                          h0=to_f64(h0), prevBx0=to_f64(u0), angle0=to_f64(a0), dh=to_f64(adj["dh_final"]),
                          dprevBx=to_f64(adj["dprevBx_final"]), dangle=to_f64(adj["dangle_final"]))
    errs = {k: relerr(v.reshape(ref[NAME.get(k, k)].shape), ref[NAME.get(k, k)]) for k, v in got.items()}
    bad = {k: e for k, e in errs.items() if not e <= BWD_TOL}
    assert not bad, (bad, errs)
