"""GPU parity of the backward (m3_chunked_bwd) against the oracle's reverse
sweep, which is itself pinned by finite differences (marked gpu).

Every gradient the call returns is compared element by element (normwise max
relative error) with the fp64 oracle on the same stored inputs.  The kernels
compute in fp32 from the stored values (bf16 inputs are widened, never
rounded again), so the bar is the fp32 one for both input dtypes: 1e-4,
which leaves room for fp32 sums over up to T*N*P products in the shared
parameters' gradients.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import cuda, norm_dev, norm_f64, relerr
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.inputs import to_f64

pytestmark = pytest.mark.gpu

SCAN = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
TOL = 1e-4
NAME = {"dW_x": "dWx", "dW_y": "dWy"}


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
    oracle.build_oracle()


def _seeded(shape, seed, scale=1.0, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * scale).to(dtype)


def _case(inp, chunk, mimo, with_state, seeds, seed=0):
    Bt, T, H, P = inp["x"].shape
    N, K = inp["B"].shape[-1], inp["theta"].shape[-1]
    st = {}
    if with_state:
        st["h0"] = _seeded((Bt, H, N, P), seed + 1, 0.5)
        st["prevBx0"] = _seeded((Bt, H, N, P), seed + 2, 0.2)
        st["angle0"] = _seeded((Bt, H, K), seed + 3, 2.0)
    dy = _seeded((Bt, T, H, P), seed + 4, 1.0, inp["x"].dtype)
    adj = {}
    if seeds:
        adj["dh_final"] = _seeded((Bt, H, N, P), seed + 5, 0.3)
        adj["dprevBx_final"] = _seeded((Bt, H, N, P), seed + 6, 0.3)
        adj["dangle_final"] = _seeded((Bt, H, K), seed + 7, 0.3)
    d = cuda(inp)
    kw = {k: v.cuda() for k, v in st.items()}
    kw.update({k: v.cuda() for k, v in adj.items()})
    if mimo:
        kw["W_x"], kw["W_y"] = d["Wx"], d["Wy"]
    got = m3.chunked_bwd(*[d[k] for k in SCAN], dy.cuda(), chunk, norm=norm_dev(inp), want=m3.GRAD_FIELDS, **kw)
    torch.cuda.synchronize()
    ref = oracle.loop_bwd(**{k: to_f64(inp[k]) for k in SCAN}, dy=to_f64(dy),
                          Wx=to_f64(inp["Wx"]) if mimo else None, Wy=to_f64(inp["Wy"]) if mimo else None,
                          norm=norm_f64(inp), **{k: to_f64(v) for k, v in st.items()},
                          dh=to_f64(adj["dh_final"]) if seeds else None,
                          dprevBx=to_f64(adj["dprevBx_final"]) if seeds else None,
                          dangle=to_f64(adj["dangle_final"]) if seeds else None)
    errs = {}
    for k, v in got.items():
        r = ref[NAME.get(k, k)]
        if k == "dangle0" and not with_state and not seeds:
            # from a zero state y depends only on angle differences (rotation
            # invariance), so this gradient is zero: compare it on the scale of
            # the angle gradients instead of its own
            scale = float(np.max(np.abs(ref["dtheta"]))) if ref["dtheta"].size else 1.0
            errs[k] = float(np.max(np.abs(v.cpu().double().numpy()))) / max(scale, 1e-30) if v.numel() else 0.0
            continue
        errs[k] = relerr(v.reshape(r.shape), r)
    return errs


def _assert(errs, tol=TOL):
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,chunk", [(1, 8), (8, 8), (9, 8), (37, 8), (70, 16)])
def test_bwd_siso_small(dtype, T, chunk):
    inp = gen.scan_inputs(2, T, 3, 8, 6, dtype=dtype, seed=600 + T + chunk)
    _assert(_case(inp, chunk, False, True, True, seed=T))


@pytest.mark.parametrize("dtype,R", [("bf16", 1), ("f32", 1), ("bf16", 2)])
def test_bwd_odd_headdim(dtype, R):
    # P = 5: rows that are not whole 4-byte words in bf16 (copied without cp.async)
    inp = gen.scan_inputs(2, 23, 2, 5, 6, rank=R, dtype=dtype, seed=605 + R, mimo_weights=R > 1)
    _assert(_case(inp, 8, R > 1, True, True, seed=11))


def test_bwd_siso_no_state_no_seeds():
    inp = gen.scan_inputs(2, 40, 2, 8, 8, dtype="f32", seed=610)
    _assert(_case(inp, 16, False, False, False, seed=3))


def test_bwd_siso_norm_bias_groups_partial():
    inp = gen.scan_inputs(2, 45, 4, 8, 16, dtype="f32", seed=611, bcnorm=True, ngroups=2, rope_pairs=3)
    _assert(_case(inp, 16, False, True, True, seed=4))


@pytest.mark.parametrize("R,G,K", [(2, 1, 3), (4, 2, 4), (3, 3, 1)])
def test_bwd_mimo(R, G, K):
    inp = gen.scan_inputs(2, 33, 6, 8, 8, rank=R, dtype="f32", seed=620 + R, bcnorm=True, ngroups=G,
                          rope_pairs=K)
    _assert(_case(inp, 8, True, True, True, seed=R))


@pytest.mark.parametrize("T", [150, 300])
def test_bwd_layer_shape_bf16(T):
    # the workloads' head shape: P 64, N 128
    inp = gen.scan_inputs(2, T, 2, 64, 128, dtype="bf16", seed=630 + T)
    _assert(_case(inp, 64, False, True, True, seed=T))


def test_bwd_mimo_layer_shape_bf16():
    inp = gen.scan_inputs(1, 70, 2, 64, 128, rank=4, dtype="bf16", seed=640, ngroups=1, rope_pairs=32)
    _assert(_case(inp, 64, True, True, True, seed=5))


def test_bwd_empty_sequence_passes_adjoints_through():
    inp = gen.scan_inputs(2, 0, 2, 8, 6, dtype="f32", seed=650)
    errs = _case(inp, 8, False, True, True, seed=9)
    for k in ("dh0", "dprevBx0", "dangle0"):
        assert errs[k] <= 1e-7, errs


def test_bwd_deterministic():
    inp = gen.scan_inputs(2, 100, 4, 16, 16, rank=2, dtype="bf16", seed=660, bcnorm=True, ngroups=2)
    d = cuda(inp)
    dy = _seeded((2, 100, 4, 16), 1, 1.0, torch.bfloat16).cuda()
    outs = [m3.chunked_bwd(*[d[k] for k in SCAN], dy, 16, W_x=d["Wx"], W_y=d["Wy"], norm=norm_dev(inp))
            for _ in range(2)]
    for k in outs[0]:
        assert torch.equal(outs[0][k], outs[1][k]), k


def test_bwd_full_size_sampled_lanes():
    """8 x 2048 x 16 heads (the default workload's shape): the per-lane
    gradients of sampled (b, h) lanes against the oracle run on those lanes."""
    Bt, T, H, P, N = 8, 2048, 16, 64, 128
    inp = gen.scan_inputs(Bt, T, H, P, N, dtype="bf16", seed=670)
    d = cuda(inp)
    dy = _seeded((Bt, T, H, P), 671, 1.0, torch.bfloat16)
    got = m3.chunked_bwd(*[d[k] for k in SCAN], dy.cuda(), 64,
                         want=("dx", "ddt", "dlam", "dtheta", "dB", "dC", "dh0", "dprevBx0", "dangle0"))
    torch.cuda.synchronize()
    for b, h in [(0, 0), (Bt - 1, H - 1), (3, 7)]:
        lane = {k: to_f64(inp[k][b:b + 1, :, h:h + 1]) for k in ("x", "dt", "lam", "theta", "B", "C")}
        lane["A"], lane["D"] = to_f64(inp["A"][h:h + 1]), to_f64(inp["D"][h:h + 1])
        ref = oracle.loop_bwd(**lane, dy=to_f64(dy[b:b + 1, :, h:h + 1]))
        for k in ("dx", "ddt", "dlam", "dtheta", "dB", "dC"):
            assert relerr(got[k][b:b + 1, :, h:h + 1], ref[k]) <= TOL, (k, b, h)
        for k in ("dh0", "dprevBx0"):
            assert relerr(got[k][b:b + 1, h:h + 1], ref[k]) <= TOL, (k, b, h)
        # from a zero state the angle gradient is zero (rotation invariance)
        scale = float(np.max(np.abs(ref["dtheta"])))
        assert float(got["dangle0"][b, h].abs().max()) <= TOL * scale, (b, h)
