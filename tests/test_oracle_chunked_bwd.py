"""Pin of the oracle's chunked backward (CPU only): the chunked reverse walk
(oracle/chunked_bwd.py) equals the loop's reverse sweep, which finite
differences pin, for every gradient, every chunk length (including 1 and
chunks longer than the sequence), ragged tails, grouped B/C, partial RoPE,
rank R with W_x and W_y, initial states and final-state adjoints.  Both are fp64, so they agree to
rounding (1e-11 relative)."""
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
