"""Pin of the oracle's chunked backward (CPU only): the chunked reverse walk
(oracle/chunked_bwd.py) equals the loop's reverse sweep, which finite
differences pin, for every gradient, every chunk length (including 1 and
chunks longer than the sequence), ragged tails, grouped B/C, partial RoPE,
rank R with W_x and W_y, initial states and final-state adjoints.  Both are fp64, so they agree to
rounding (1e-11 relative).  Nine plausible mistakes planted in a copy of the
chunked walk each break that agreement, so the pin constrains every term."""
import numpy as np
import pytest

import oracle
from oracle.chunked_bwd import chunked_bwd

KEYS = ("dx", "ddt", "dA", "dlam", "dtheta", "dB", "dC", "dD", "dh0", "dprevBx0", "dangle0")


def _case(seed, Bt, T, H, G, P, N, K, states, shift=-1.0):
    rng = np.random.default_rng(seed)
    sp = lambda v: np.log1p(np.exp(v))
    inp = dict(x=rng.standard_normal((Bt, T, H, P)), dt=sp(rng.standard_normal((Bt, T, H)) + shift),
               A=-np.exp(rng.uniform(0, 1, H)), lam=1 / (1 + np.exp(-rng.standard_normal((Bt, T, H)))),
               theta=rng.uniform(-1.0, 1.0, (Bt, T, H, K)), B=rng.standard_normal((Bt, T, G, N)) / np.sqrt(N),
               C=rng.standard_normal((Bt, T, G, N)) / np.sqrt(N), D=rng.standard_normal(H))
    dy = rng.standard_normal((Bt, T, H, P))
    st, adj = {}, {}
    if states:
        st = dict(h0=0.5 * rng.standard_normal((Bt, H, N, P)), prevBx0=0.3 * rng.standard_normal((Bt, H, N, P)),
                  angle0=rng.uniform(-3, 3, (Bt, H, K)))
        adj = dict(dh=0.3 * rng.standard_normal((Bt, H, N, P)), dprevBx=0.3 * rng.standard_normal((Bt, H, N, P)),
                   dangle=0.3 * rng.standard_normal((Bt, H, K)))
    return inp, dy, st, adj


def _rel(g, r):
    g, r = np.asarray(g, float), np.asarray(r, float)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))


@pytest.fixture(scope="module", autouse=True)
def _build():
    oracle.build_oracle()


@pytest.mark.parametrize("T,Q", [(1, 1), (5, 1), (37, 4), (37, 16), (64, 16), (70, 64), (20, 100)])
@pytest.mark.parametrize("states", [False, True])
def test_chunked_backward_equals_the_loop(T, Q, states):
    inp, dy, st, adj = _case(11 + T + Q, 2, T, 2, 2, 5, 6, 3, states)
    ref = oracle.loop_bwd(**inp, dy=dy, **st, **adj)
    got = chunked_bwd(**inp, dy=dy, chunk=Q, **st, **adj)
    if T == 1 and not states:
        # one token from zero states: y_0 holds Cbar_0 . Bbar_0, which no
        # rotation changes, so every angle gradient is zero on both sides
        for k in ("dtheta", "dangle0"):
            assert float(np.max(np.abs(got[k]))) <= 1e-12 and float(np.max(np.abs(ref[k]))) <= 1e-12
    skip = ("dangle0", "dtheta") if T == 1 and not states else ("dangle0",)
    errs = {k: _rel(got[k], ref[k]) for k in KEYS if k not in skip}
    assert max(errs.values()) <= 1e-11, errs
    if T == 1 and not states:
        return
    if states:
        assert _rel(got["dangle0"], ref["dangle0"]) <= 1e-11
    else:
        # from zero states y depends on angle differences only, so the angle0
        # gradient is zero: both sides hold rounding noise on the dtheta scale
        scale = float(np.max(np.abs(ref["dtheta"])))
        assert float(np.max(np.abs(got["dangle0"] - ref["dangle0"]))) <= 1e-11 * scale


@pytest.mark.parametrize("H,G,K", [(4, 1, 2), (6, 3, 1), (4, 2, 4)])
def test_chunked_backward_groups_and_partial_rope(H, G, K):
    inp, dy, st, adj = _case(5 * H + G + K, 1, 45, H, G, 4, 8, K, True)
    ref = oracle.loop_bwd(**inp, dy=dy, **st, **adj)
    got = chunked_bwd(**inp, dy=dy, chunk=8, **st, **adj)
    errs = {k: _rel(got[k], ref[k]) for k in KEYS}
    assert max(errs.values()) <= 1e-11, errs


def test_chunked_backward_strong_decay():
    """Long steps (dt around 5) drive the in-chunk decays to underflow; the
    chunked walk still agrees with the loop."""
    inp, dy, st, adj = _case(3, 1, 90, 2, 2, 4, 6, 3, True, shift=5.0)
    ref = oracle.loop_bwd(**inp, dy=dy, **st, **adj)
    got = chunked_bwd(**inp, dy=dy, chunk=32, **st, **adj)
    errs = {k: _rel(got[k], ref[k]) for k in KEYS}
    assert max(errs.values()) <= 1e-11, errs


@pytest.mark.parametrize("R,G,K,T,Q,states", [(2, 2, 3, 37, 8, True), (3, 1, 2, 20, 4, True), (4, 2, 4, 33, 16, False),
                                              (2, 2, 1, 9, 1, True)])
def test_chunked_backward_rank_r(R, G, K, T, Q, states):
    """Rank R: the walk over (token, rank) rows with W_x, W_y equals the loop,
    including the W_x and W_y gradients."""
    H, P, N = 2, 4, 8
    inp, dy, st, adj = _case(100 * R + T, 1, T, H, G, P, N, K, states)
    rng = np.random.default_rng(R + T)
    inp["B"] = rng.standard_normal((1, T, G, R, N)) / np.sqrt(N)
    inp["C"] = rng.standard_normal((1, T, G, R, N)) / np.sqrt(N)
    W = dict(Wx=1 + 0.3 * rng.standard_normal((H, R, P)), Wy=1 + 0.3 * rng.standard_normal((H, R, P)))
    ref = oracle.loop_bwd(**inp, dy=dy, **W, **st, **adj)
    got = chunked_bwd(**inp, dy=dy, chunk=Q, **W, **st, **adj)
    keys = KEYS + ("dWx", "dWy")
    errs = {k: _rel(got[k], ref[k]) for k in keys if states or k != "dangle0"}
    assert max(errs.values()) <= 1e-11, errs


CHUNKED_MUTATIONS = [
    ("inter-chunk decay of the adjoint state dropped", "dgin = dgin + np.exp(ce) * Gout", "dgin = dgin + Gout"),
    ("mask diagonal takes w instead of gamma", "M = E * wc[None, :] + np.diag(gc)",
     "M = E * wc[None, :] + np.diag(wc)"),
    ("chunk-state weight without the decay", "sc = rows(es * wc)", "sc = rows(wc)"),
    ("decay adjoint of the chunk-state weights dropped", "        dcum -= des\n", "\n"),
    ("rotation adjoint sign", "dphi += cross.reshape(T, R, K).sum(axis=1)", "dphi -= cross.reshape(T, R, K).sum(axis=1)"),
    ("angle adjoint summed forwards", "rc = np.cumsum(dphi[::-1], axis=0)[::-1]", "rc = np.cumsum(dphi, axis=0)"),
    ("boundary fold adjoint dropped", "    ddt[0] += (1.0 - lam[0]) * dsg_m1\n", "\n"),
    ("prevBx_final adjoint from the wrong token", "last = slice((T - 1) * R, T * R)", "last = slice(0, R)"),
    ("W_y gradient without the inter-chunk term", "Y = rows(ec)[:, None] * (Cc @ gi) + (Mr * S) @ Xc",
     "Y = (Mr * S) @ Xc"),
]


@pytest.mark.parametrize("name,old,new", CHUNKED_MUTATIONS, ids=[m[0] for m in CHUNKED_MUTATIONS])
def test_planted_mistakes_in_the_chunked_backward_fail_the_pin(name, old, new):
    """Each plausible mistake planted in a copy of the chunked walk makes it
    disagree with the loop on one of the pin's cases."""
    import os
    import types
    src = open(os.path.join(os.path.dirname(oracle.__file__), "chunked_bwd.py")).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType("mutated_chunked_bwd")
    exec(compile(src.replace(old, new), "mutated_chunked_bwd", "exec"), mod.__dict__)
    worst = 0.0
    for R in (1, 2):
        inp, dy, st, adj = _case(7 + R, 1, 23, 2, 2, 4, 6, 2, True)
        kw = {}
        if R > 1:
            rng = np.random.default_rng(R)
            inp["B"] = rng.standard_normal((1, 23, 2, R, 6)) / np.sqrt(6)
            inp["C"] = rng.standard_normal((1, 23, 2, R, 6)) / np.sqrt(6)
            kw = dict(Wx=1 + 0.3 * rng.standard_normal((2, R, 4)), Wy=1 + 0.3 * rng.standard_normal((2, R, 4)))
        ref = oracle.loop_bwd(**inp, dy=dy, **kw, **st, **adj)
        got = mod.chunked_bwd(**inp, dy=dy, chunk=5, **kw, **st, **adj)
        worst = max([worst] + [_rel(got[k], ref[k]) for k in got])
    assert worst > 1e-6, name
