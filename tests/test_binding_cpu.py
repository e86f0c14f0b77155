"""The Python binding checks every tensor against the sizes it passes in
m3_dims (element count, dtype, device) before any call, so a short buffer
can never reach a kernel (CPU only: every call here stops in the binding)."""
import pytest
import torch

from state_space_lm_b200 import build as m3build
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3

SCAN = ("x", "dt", "A", "lam", "theta", "B", "C", "D")


@pytest.fixture(scope="module", autouse=True)
def built():
    m3build.build()


def _cut(t):
    """One row short along the first axis: the mistake the checks exist for."""
    return t[:-1].clone()


def _reaches_the_library(fn):
    # past the binding's checks the first thing that fails on a CPU tensor is
    # the pointer marshalling, which wants CUDA memory
    with pytest.raises(ValueError, match="expected a CUDA tensor"):
        fn()


@pytest.mark.parametrize("mimo", [False, True])
def test_scan_forward_and_backward_checks(mimo):
    inp = gen.scan_inputs(2, 12, 4, 8, 16, rank=2 if mimo else 1, dtype="bf16", seed=3, mimo_weights=mimo,
                          bcnorm=True, ngroups=2, rope_pairs=6)
    fwd = m3.mimo_chunked_fwd if mimo else m3.siso_chunked_fwd
    nrm = {k: inp[k] for k in ("normw_B", "normw_C", "bias_B", "bias_C")}
    kw = dict(norm=nrm, **({"W_x": inp["Wx"], "W_y": inp["Wy"]} if mimo else {}))
    args = [inp[k] for k in SCAN]
    dy = gen.grad_seed(inp["x"], 4)
    _reaches_the_library(lambda: fwd(*args, 4, **kw))
    _reaches_the_library(lambda: m3.chunked_bwd(*args, dy, 4, **kw))
    for i, name in enumerate(SCAN):
        if name in ("x",):
            continue                                   # x defines the sizes
        bad = list(args)
        bad[i] = _cut(args[i])
        with pytest.raises(ValueError, match=r": %s(_t)? (has|is) " % name):
            fwd(*bad, 4, **kw)
        with pytest.raises(ValueError, match=r": %s(_t)? (has|is) " % name):
            m3.chunked_bwd(*bad, dy, 4, **kw)
    # wrong dtypes: fp32 B under bf16 x, bf16 dt
    bad = list(args)
    bad[5] = args[5].float()
    with pytest.raises(ValueError, match="B is torch.float32"):
        fwd(*bad, 4, **kw)
    bad = list(args)
    bad[1] = args[1].bfloat16()
    with pytest.raises(ValueError, match="dt is torch.bfloat16"):
        fwd(*bad, 4, **kw)
    # optional states and norm parameters are checked when given
    Bt, T, H, P = inp["x"].shape
    N, K = inp["B"].shape[-1], inp["theta"].shape[-1]
    with pytest.raises(ValueError, match="h0"):
        fwd(*args, 4, h0=torch.zeros(Bt, H, N, P - 1), **kw)
    with pytest.raises(ValueError, match="angle0"):
        fwd(*args, 4, angle0=torch.zeros(Bt, H, K + 1), **kw)
    with pytest.raises(ValueError, match="bias_C"):
        fwd(*args, 4, **{**kw, "norm": {**nrm, "bias_C": _cut(nrm["bias_C"])}})
    with pytest.raises(ValueError, match="dh_final"):
        m3.chunked_bwd(*args, dy, 4, dh_final=torch.zeros(Bt, H, N + 2, P), **kw)
    with pytest.raises(ValueError, match="dy"):
        m3.chunked_bwd(*args, _cut(dy), 4, **kw)
    with pytest.raises(ValueError, match="dx"):
        m3.chunked_bwd(*args, dy, 4, out={"dx": torch.empty(Bt, T, H, P + 1)}, **kw)
    if mimo:
        with pytest.raises(ValueError, match="W_y"):
            fwd(*args, 4, **{**kw, "W_y": _cut(inp["Wy"])})
    # preallocated outputs of the wrong size or dtype
    y = torch.empty(Bt, T, H, P, dtype=torch.float32)
    h = torch.empty(Bt, H, N, P)
    with pytest.raises(ValueError, match="y has"):
        fwd(*args, 4, out=(_cut(y).bfloat16(), h, h.clone(), torch.empty(Bt, H, K)), **kw)
    with pytest.raises(ValueError, match="y is torch.float32"):
        fwd(*args, 4, out=(y, h, h.clone(), torch.empty(Bt, H, K)), **kw)


def test_decode_checks():
    g = gen.make_generator(5)
    Bt, H, P, N, R, G, K = 3, 4, 8, 16, 2, 2, 6
    st = gen.decode_step_inputs(g, Bt, H, P, N, rank=R, ngroups=G, rope_pairs=K)
    A, D = torch.randn(H), torch.randn(H)
    h, u, a = torch.zeros(Bt, H, N, P), torch.zeros(Bt, H, N, P), torch.zeros(Bt, H, K)
    bp, xp = torch.zeros(Bt, H, R, N), torch.zeros(Bt, H, P)
    args = lambda s: (s["x"], s["dt"], A, s["lam"], s["theta"], s["B"], s["C"], D)
    _reaches_the_library(lambda: m3.mimo_step_decode(*args(st), h, u, a))
    _reaches_the_library(lambda: m3.step_decode_factored(*args(st), h, bp, xp, a))
    for name in ("dt", "lam", "theta", "B", "C"):
        bad = dict(st, **{name: _cut(st[name])})
        with pytest.raises(ValueError, match=r": %s(_t)? (has|is) " % name):
            m3.mimo_step_decode(*args(bad), h, u, a)
        with pytest.raises(ValueError, match=r": %s(_t)? (has|is) " % name):
            m3.step_decode_factored(*args(bad), h, bp, xp, a)
    with pytest.raises(ValueError, match="prevBx"):
        m3.mimo_step_decode(*args(st), h, _cut(u), a)
    with pytest.raises(ValueError, match="h has"):
        m3.step_decode_factored(*args(st), _cut(h), bp, xp, a)
    with pytest.raises(ValueError, match="b_prev"):
        m3.step_decode_factored(*args(st), h, _cut(bp), xp, a)
    with pytest.raises(ValueError, match="x_prev is torch.bfloat16"):
        m3.step_decode_factored(*args(st), h, bp, xp.bfloat16(), a)
    with pytest.raises(ValueError, match="angle"):
        m3.step_decode_factored(*args(st), h, bp, xp, _cut(a))
    with pytest.raises(ValueError, match="y_t"):
        m3.mimo_step_decode(*args(st), h, u, a, y_out=torch.empty(Bt, H, P + 1, dtype=torch.bfloat16))
    # the SISO step: B_t (Bt, G, N)
    s1 = gen.decode_step_inputs(g, Bt, H, P, N, ngroups=G, rope_pairs=K)
    _reaches_the_library(lambda: m3.step_decode(*args(s1), h, u, a))
    with pytest.raises(ValueError, match="C_t"):
        m3.step_decode(*args(dict(s1, C=_cut(s1["C"]))), h, u, a)
    with pytest.raises(ValueError, match="A has"):
        m3.step_decode(s1["x"], s1["dt"], A[:-1], s1["lam"], s1["theta"], s1["B"], s1["C"], D, h, u, a)


def test_rope_and_discretize_checks():
    inp = gen.scan_inputs(2, 5, 4, 8, 16, dtype="f32", seed=6, ngroups=2, rope_pairs=5)
    _reaches_the_library(lambda: m3.rope_bc(inp["B"], inp["C"], inp["theta"], inp["dt"]))
    with pytest.raises(ValueError, match="theta"):
        m3.rope_bc(inp["B"], inp["C"], _cut(inp["theta"]), inp["dt"])
    with pytest.raises(ValueError, match="C is torch.bfloat16"):
        m3.rope_bc(inp["B"], inp["C"].bfloat16(), inp["theta"], inp["dt"])
    with pytest.raises(ValueError, match="angle0"):
        m3.rope_bc(inp["B"], inp["C"], inp["theta"], inp["dt"], angle0=torch.zeros(2, 4, 4))
    _reaches_the_library(lambda: m3.discretize(inp["dt"], inp["A"], inp["lam"]))
    with pytest.raises(ValueError, match="lam"):
        m3.discretize(inp["dt"], inp["A"], _cut(inp["lam"]))
    with pytest.raises(ValueError, match="A has"):
        m3.discretize(inp["dt"], torch.zeros(5), inp["lam"])
    with pytest.raises(ValueError, match="float32 or bfloat16"):
        m3.siso_chunked_fwd(inp["x"].double(), *[inp[k] for k in SCAN[1:]], 4)
