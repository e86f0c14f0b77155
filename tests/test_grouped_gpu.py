"""GPU parity for grouped B/C and partial RoPE (marked gpu).

Head h reads the B/C row of group h / (H / G) (TorchMamba README, "Models":
n_groups with H % G == 0), and only the first K pairs of B and C rotate
(dotLLM pull request, real-checkpoint run: num_rope_angles 32 of d_state
128).  Every entry point is compared with the fp64 oracle on the same seeded
inputs: the tensor-core scan (K a multiple of 4), the FFMA scan (fp32, or K
not a multiple of 4), the segmented long-sequence path, the standalone RoPE
and the three decode steps.  Bars as in the other parity tests: 1e-5 for fp32
inputs, 2e-2 for bf16 inputs (max relative error, normwise).
"""
import pytest
import torch

import oracle
from helpers import TOL, cuda, norm_dev, norm_f64, relerr
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.inputs import to_f64

pytestmark = pytest.mark.gpu

SCAN = ("x", "dt", "A", "lam", "theta", "B", "C", "D")


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
    oracle.build_oracle()


def _states(Bt, H, N, P, K, seed):
    g = torch.Generator().manual_seed(seed)
    h0 = torch.randn(Bt, H, N, P, generator=g, dtype=torch.float64).float() * 0.5
    u0 = torch.randn(Bt, H, N, P, generator=g, dtype=torch.float64).float() * 0.1
    a0 = (torch.rand(Bt, H, K, generator=g, dtype=torch.float64) * 6 - 3).float()
    return h0, u0, a0


def _chunked(inp, chunk, mimo, with_state, seed=0):
    Bt, T, H, P = inp["x"].shape
    N, K = inp["B"].shape[-1], inp["theta"].shape[-1]
    st = _states(Bt, H, N, P, K, seed) if with_state else (None, None, None)
    d = cuda(inp)
    dev = [None if s is None else s.cuda() for s in st]
    args = [d[k] for k in SCAN]
    kw = dict(norm=norm_dev(inp), h0=dev[0], prevBx0=dev[1], angle0=dev[2])
    if mimo:
        got = m3.mimo_chunked_fwd(*args, chunk, W_x=d.get("Wx"), W_y=d.get("Wy"), **kw)
    else:
        got = m3.siso_chunked_fwd(*args, chunk, **kw)
    torch.cuda.synchronize()
    ref_args = {k: to_f64(inp[k]) for k in SCAN}
    rkw = dict(h0=None if st[0] is None else to_f64(st[0]), prevBx0=None if st[1] is None else to_f64(st[1]),
               angle0=None if st[2] is None else to_f64(st[2]), norm=norm_f64(inp))
    if mimo:
        ref = oracle.mimo_loop(**ref_args, Wx=to_f64(inp["Wx"]), Wy=to_f64(inp["Wy"]), **rkw)
    else:
        ref = oracle.siso_loop(**ref_args, **rkw)
    assert got[3].shape == (Bt, H, K)
    return [relerr(g, r) for g, r in zip(got, ref)]


# ----------------------------------------------------------------------------
# S2 standalone RoPE
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("H,G,R,N,K,bcnorm", [(4, 1, 1, 16, 3, True), (6, 3, 3, 8, 4, False),
                                              (8, 2, 1, 128, 32, True), (4, 4, 4, 128, 1, False)])
def test_rope_grouped_partial(dtype, H, G, R, N, K, bcnorm):
    inp = gen.scan_inputs(2, 45, H, 4, N, rank=R, dtype=dtype, seed=300 + N + K, mimo_weights=R > 1,
                          bcnorm=bcnorm, ngroups=G, rope_pairs=K)
    a0 = _states(2, H, N, 4, K, 7)[2]
    d = cuda(inp)
    Br, Cr, ang = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"], angle0=a0.cuda(), norm=norm_dev(inp))
    rB, rC, rA = oracle.rope_bc(to_f64(inp["B"]), to_f64(inp["C"]), to_f64(inp["theta"]), to_f64(inp["dt"]),
                                angle0=to_f64(a0), norm=norm_f64(inp))
    tol = TOL[gen.storage_dtype(dtype)]
    assert Br.shape == rB.shape and ang.shape == (2, H, K)
    assert relerr(Br, rB) <= tol
    assert relerr(Cr, rC) <= tol
    assert relerr(ang, rA) <= 1e-5


# ----------------------------------------------------------------------------
# chunked forwards
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("G,K,T", [(1, 32, 150), (2, 64, 130), (4, 16, 64), (1, 4, 77), (8, 32, 1)])
def test_siso_tc_grouped_partial(G, K, T):
    inp = gen.scan_inputs(2, T, 8, 64, 128, dtype="bf16", seed=310 + G + K + T, ngroups=G, rope_pairs=K)
    errs = _chunked(inp, 64, False, True, seed=G + K)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


def test_siso_tc_grouped_partial_norm_bias():
    inp = gen.scan_inputs(2, 200, 4, 64, 128, dtype="bf16", seed=320, bcnorm=True, ngroups=1, rope_pairs=32)
    errs = _chunked(inp, 128, False, True, seed=3)
    assert max(errs) <= 2e-2, errs


@pytest.mark.parametrize("G,K", [(1, 30), (2, 3)])
def test_siso_bf16_pairs_not_multiple_of_4(G, K):
    # the tensor-core kernel loads theta 4 pairs at a time; these take the FFMA path
    inp = gen.scan_inputs(2, 90, 4, 64, 128, dtype="bf16", seed=330 + K, ngroups=G, rope_pairs=K)
    errs = _chunked(inp, 64, False, True, seed=K)
    assert max(errs) <= 2e-2, errs


@pytest.mark.parametrize("G,K,bcnorm", [(1, 3, False), (3, 8, True), (6, 1, True)])
def test_siso_fp32_grouped_partial(G, K, bcnorm):
    inp = gen.scan_inputs(2, 70, 6, 8, 16, dtype="f32", seed=340 + G + K, bcnorm=bcnorm, ngroups=G, rope_pairs=K)
    errs = _chunked(inp, 16, False, True, seed=G)
    assert max(errs) <= 1e-5, errs


@pytest.mark.parametrize("Bt,H,G,T", [(1, 2, 1, 3000), (2, 4, 2, 2600)])
def test_siso_tc_segmented_grouped_partial(Bt, H, G, T):
    # few lanes: the sequence is cut into segments chained by the combine kernel
    inp = gen.scan_inputs(Bt, T, H, 64, 128, dtype="bf16", dt_shift=-4.0, seed=350 + T, ngroups=G,
                          rope_pairs=32)
    errs = _chunked(inp, 64, False, True, seed=T)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


@pytest.mark.parametrize("R,G,K,T", [(2, 2, 32, 130), (4, 1, 32, 100), (4, 4, 8, 70)])
def test_mimo_tc_grouped_partial(R, G, K, T):
    inp = gen.scan_inputs(2, T, 4, 64, 128, rank=R, dtype="bf16", seed=360 + R + G + K, ngroups=G,
                          rope_pairs=K)
    errs = _chunked(inp, 64, True, True, seed=R)
    assert max(errs) <= 2e-2, errs
    assert m3.device_error() == m3.M3_OK


def test_mimo_fp32_grouped_partial():
    inp = gen.scan_inputs(2, 40, 6, 8, 16, rank=3, dtype="f32", seed=370, bcnorm=True, ngroups=2, rope_pairs=5)
    errs = _chunked(inp, 8, True, True, seed=1)
    assert max(errs) <= 1e-5, errs


# ----------------------------------------------------------------------------
# decode steps after a prefill
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("form,R,G,K,dtype", [("siso", 1, 2, 32, "bf16"), ("siso", 1, 1, 3, "f32"),
                                              ("mimo", 2, 1, 16, "bf16"), ("mimo", 4, 3, 5, "f32"),
                                              ("mimo", 4, 2, 64, "bf16"),
                                              ("factored", 1, 2, 32, "bf16"), ("factored", 4, 1, 32, "bf16"),
                                              ("factored", 2, 3, 64, "bf16"), ("factored", 3, 1, 16, "bf16"),
                                              ("factored", 3, 3, 2, "f32")])
def test_decode_grouped_partial(form, R, G, K, dtype):
    Bt, T0, H, P, N, steps = 3, 20, 6, 8, 16, 6
    if dtype == "bf16":
        P, N = 64, 128
    mimo = form != "siso" and (R > 1 or form == "mimo")
    inp = gen.scan_inputs(Bt, T0, H, P, N, rank=R, dtype=dtype, seed=380 + R + G + K, mimo_weights=mimo,
                          ngroups=G, rope_pairs=K)
    if form == "factored" and not mimo:
        inp["B"], inp["C"] = inp["B"][:, :, :, None], inp["C"][:, :, :, None]
        mimo = True
    g = inp.pop("generator")
    toks = [gen.decode_step_inputs(g, Bt, H, P, N, dtype=dtype, rank=R, rank_axis=mimo, ngroups=G,
                                   rope_pairs=K) for _ in range(steps)]
    Wx = inp.get("Wx", torch.ones(H, R, P))
    Wy = inp.get("Wy", torch.ones(H, R, P))
    # the whole sequence by the oracle loop
    per_token = ("x", "dt", "lam", "theta", "B", "C")
    full = {k: (torch.cat([inp[k]] + [t[k][:, None] for t in toks], 1) if k in per_token else inp[k])
            for k in SCAN}
    rf = {k: to_f64(v) for k, v in full.items()}
    ref = (oracle.mimo_loop(**rf, Wx=to_f64(Wx), Wy=to_f64(Wy)) if mimo else oracle.siso_loop(**rf))
    # prefill by the oracle (the state handed to the decode steps), then GPU steps
    pre = {k: to_f64(inp[k]) for k in SCAN}
    if mimo:
        _, h, u, a = oracle.mimo_loop(**pre, Wx=to_f64(Wx), Wy=to_f64(Wy))
    else:
        _, h, u, a = oracle.siso_loop(**pre)
    h = torch.from_numpy(h).float().cuda()
    u = torch.from_numpy(u).float().cuda()
    a = torch.from_numpy(a).float().cuda()
    if form == "factored":
        Br, _, _ = oracle.rope_bc(pre["B"], pre["C"], pre["theta"], pre["dt"])
        bp = torch.from_numpy(Br[:, -1]).float().cuda().contiguous()
        xp = inp["x"][:, -1].float().cuda().contiguous()
    dA, dD, dWx, dWy = inp["A"].cuda(), inp["D"].cuda(), Wx.cuda(), Wy.cuda()
    tol = TOL[gen.storage_dtype(dtype)]
    for s, t in enumerate(toks):
        dt_ = cuda(t)
        args = (dt_["x"], dt_["dt"], dA, dt_["lam"], dt_["theta"], dt_["B"], dt_["C"], dD)
        if form == "siso":
            y = m3.step_decode(*args, h, u, a)
        elif form == "mimo":
            y = m3.mimo_step_decode(*args, h, u, a, W_x=dWx, W_y=dWy)
        else:
            y = m3.step_decode_factored(*args, h, bp, xp, a, W_x=dWx, W_y=dWy)
        torch.cuda.synchronize()
        assert relerr(y, ref[0][:, T0 + s]) <= tol, s
    assert relerr(h, ref[1]) <= tol
    assert relerr(a, ref[3]) <= 1e-5


# ----------------------------------------------------------------------------
# full-size workload, sampled lanes: 8 x 2048 x 16 heads, one B/C group, 32
# rotated pairs of 64 (the 370M checkpoint's rope fraction 0.5)
# ----------------------------------------------------------------------------
def test_full_size_grouped_partial_sampled_lanes():
    Bt, T, H, P, N, G, K = 8, 2048, 16, 64, 128, 1, 32
    inp = gen.scan_inputs(Bt, T, H, P, N, dtype="bf16", seed=390, ngroups=G, rope_pairs=K)
    d = cuda(inp)
    y, hf, uf, af = m3.siso_chunked_fwd(*[d[k] for k in SCAN], 64)
    torch.cuda.synchronize()
    assert m3.device_error() == m3.M3_OK
    for b, h in [(0, 0), (Bt - 1, H - 1), (3, 7)]:
        g = h // (H // G)
        lane = {k: to_f64(inp[k][b:b + 1, :, h:h + 1]) for k in ("x", "dt", "lam", "theta")}
        lane["B"] = to_f64(inp["B"][b:b + 1, :, g:g + 1])
        lane["C"] = to_f64(inp["C"][b:b + 1, :, g:g + 1])
        lane["A"], lane["D"] = to_f64(inp["A"][h:h + 1]), to_f64(inp["D"][h:h + 1])
        ry, rh, ru, ra = oracle.siso_loop(**lane)
        assert relerr(y[b:b + 1, :, h:h + 1], ry) <= 2e-2
        assert relerr(hf[b:b + 1, h:h + 1], rh) <= 2e-2
        assert relerr(uf[b:b + 1, h:h + 1], ru) <= 2e-2
        assert relerr(af[b:b + 1, h:h + 1], ra) <= 1e-5
