"""Pins of the oracle's backward against central finite differences of its
forward (CPU only).

The backward (the reverse sweep of the loop) is checked element by element
against (L(v + e) - L(v - e)) / 2e for every element v of every input, with
L = <dy, y> + <dh, h_final> + <du, prevBx_final> + <da, angle_final> and the
forward computed by the already-pinned loop.  Central differences of a smooth
function at e = 1e-6 in fp64 are accurate to about 1e-9 relative, far below
the 1e-6 bar used here, so a dropped term, a wrong sign or a transposed index
anywhere in the backward fails.  (Training needs these gradients: TorchMamba
README, "Models" and "Verification".)
"""
import numpy as np
import pytest

import oracle

EPS = 1e-6


def _inputs(rng, Bt, T, H, G, P, N, R, K, rank_axis, norm, state):
    sp = lambda v: np.log1p(np.exp(v))
    bc = (Bt, T, G, R, N) if rank_axis else (Bt, T, G, N)
    inp = dict(
        x=rng.standard_normal((Bt, T, H, P)),
        dt=sp(rng.standard_normal((Bt, T, H)) - 1.0),
        A=-np.exp(rng.uniform(0, 1, H)),
        lam=1 / (1 + np.exp(-rng.standard_normal((Bt, T, H)))),
        theta=rng.uniform(-1.0, 1.0, (Bt, T, H, K)),
        B=rng.standard_normal(bc) / np.sqrt(N),
        C=rng.standard_normal(bc) / np.sqrt(N),
        D=rng.standard_normal(H),
    )
    extra = {}
    if rank_axis:
        extra["Wx"] = 1 + 0.3 * rng.standard_normal((H, R, P))
        extra["Wy"] = 1 + 0.3 * rng.standard_normal((H, R, P))
    if state:
        extra["h0"] = 0.5 * rng.standard_normal((Bt, H, N, P))
        extra["prevBx0"] = 0.3 * rng.standard_normal((Bt, H, N, P))
        extra["angle0"] = rng.uniform(-3, 3, (Bt, H, K))
    nrm = None
    if norm:
        nrm = dict(normw_B=1 + 0.2 * rng.standard_normal(N), normw_C=1 + 0.2 * rng.standard_normal(N),
                   bias_B=0.3 * rng.standard_normal((H, R, N)), bias_C=0.3 * rng.standard_normal((H, R, N)),
                   eps=1e-5)
    return inp, extra, nrm


def _forward(inp, extra, nrm, rank_axis):
    if rank_axis:
        return oracle.mimo_loop(**inp, **extra, norm=nrm, nthreads=1)
    return oracle.siso_loop(**inp, **extra, norm=nrm, nthreads=1)


def _loss(outs, seeds):
    return sum(float(np.sum(o * s)) for o, s in zip(outs, seeds))


def _fd_check(inp, extra, nrm, rank_axis, seeds):
    grads = oracle.loop_bwd(**inp, **extra, norm=nrm, dy=seeds[0], dh=seeds[1], dprevBx=seeds[2],
                            dangle=seeds[3])
    targets = [(inp, k, "d" + k) for k in inp] + [(extra, k, "d" + k) for k in extra]
    if nrm is not None:
        targets += [(nrm, k, "d" + k) for k in ("normw_B", "normw_C", "bias_B", "bias_C")]
    worst = {}
    for holder, key, gname in targets:
        v = holder[key]
        fd = np.zeros_like(v)
        flat = v.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + EPS
            lp = _loss(_forward(inp, extra, nrm, rank_axis), seeds)
            flat[i] = keep - EPS
            lm = _loss(_forward(inp, extra, nrm, rank_axis), seeds)
            flat[i] = keep
            fd.reshape(-1)[i] = (lp - lm) / (2 * EPS)
        g = grads[gname]
        assert g is not None, gname
        assert g.shape == v.shape, (gname, g.shape, v.shape)
        scale = max(np.max(np.abs(fd)), 1e-3)
        worst[gname] = float(np.max(np.abs(g - fd)) / scale)
    bad = {k: e for k, e in worst.items() if e > 1e-6}
    assert not bad, bad
    return worst


def _seeds(rng, Bt, T, H, P, N, K):
    return (rng.standard_normal((Bt, T, H, P)), rng.standard_normal((Bt, H, N, P)),
            rng.standard_normal((Bt, H, N, P)), rng.standard_normal((Bt, H, K)))


@pytest.mark.parametrize("T", [1, 2, 6])
def test_siso_grad_matches_finite_differences(T):
    rng = np.random.default_rng(500 + T)
    Bt, H, P, N = 2, 2, 3, 4
    inp, extra, nrm = _inputs(rng, Bt, T, H, H, P, N, 1, N // 2, False, False, True)
    _fd_check(inp, extra, nrm, False, _seeds(rng, Bt, T, H, P, N, N // 2))


def test_siso_grad_norm_bias_groups_partial():
    rng = np.random.default_rng(510)
    Bt, T, H, G, P, N, K = 1, 5, 4, 2, 3, 8, 2
    inp, extra, nrm = _inputs(rng, Bt, T, H, G, P, N, 1, K, False, True, True)
    _fd_check(inp, extra, nrm, False, _seeds(rng, Bt, T, H, P, N, K))


@pytest.mark.parametrize("R,G,K", [(2, 1, 3), (3, 3, 1)])
def test_mimo_grad_matches_finite_differences(R, G, K):
    rng = np.random.default_rng(520 + R)
    Bt, T, H, P, N = 2, 4, 3, 2, 6
    inp, extra, nrm = _inputs(rng, Bt, T, H, G, P, N, R, K, True, True, True)
    _fd_check(inp, extra, nrm, True, _seeds(rng, Bt, T, H, P, N, K))


def test_grad_without_output_seeds_is_zero():
    rng = np.random.default_rng(530)
    inp, extra, nrm = _inputs(rng, 1, 3, 2, 2, 2, 4, 1, 2, False, False, True)
    g = oracle.loop_bwd(**inp, **extra)
    for k in oracle.GRAD_NAMES:
        if g[k] is not None:
            assert np.all(g[k] == 0.0), k
