"""The autograd wrapper's plumbing on CPU: with the library's forward and
backward replaced by the fp64 oracle (forward loop and reverse sweep),
torch.autograd.gradcheck compares the wrapper's analytic gradients -- the
backward's outputs routed to their inputs -- with finite differences of its
forward, for every input including the initial states, through all four
outputs.  A misrouted or mis-scaled gradient fails."""
import numpy as np
import pytest
import torch

import oracle
from state_space_lm_b200 import autograd as ag
from state_space_lm_b200 import m3

F = lambda t: None if t is None else t.detach().double().numpy()
T64 = lambda a: torch.from_numpy(np.ascontiguousarray(a))


def _fwd(mimo):
    def run(x, dt, A, lam, theta, B, C, D, chunk, W_x=None, W_y=None, h0=None, prevBx0=None, angle0=None, **kw):
        args = [F(v) for v in (x, dt, A, lam, theta, B, C, D)]
        st = dict(h0=F(h0), prevBx0=F(prevBx0), angle0=F(angle0))
        out = (oracle.mimo_loop(*args, Wx=F(W_x), Wy=F(W_y), **st) if mimo else oracle.siso_loop(*args, **st))
        return tuple(T64(o) for o in out)
    return run


def _bwd(x, dt, A, lam, theta, B, C, D, dy, chunk, W_x=None, W_y=None, h0=None, prevBx0=None, angle0=None,
         dh_final=None, dprevBx_final=None, dangle_final=None, want=None, **kw):
    g = oracle.loop_bwd(*[F(v) for v in (x, dt, A, lam, theta, B, C, D)], dy=F(dy), Wx=F(W_x), Wy=F(W_y),
                        h0=F(h0), prevBx0=F(prevBx0), angle0=F(angle0), dh=F(dh_final), dprevBx=F(dprevBx_final),
                        dangle=F(dangle_final))
    name = {"dW_x": "dWx", "dW_y": "dWy"}
    return {k: T64(g[name.get(k, k)]) for k in want if g.get(name.get(k, k)) is not None}


@pytest.mark.parametrize("mimo", [False, True])
def test_gradients_route_to_their_inputs(monkeypatch, mimo):
    monkeypatch.setattr(m3, "siso_chunked_fwd", _fwd(False))
    monkeypatch.setattr(m3, "mimo_chunked_fwd", _fwd(True))
    monkeypatch.setattr(m3, "chunked_bwd", _bwd)
    rng = np.random.default_rng(5 + mimo)
    Bt, T, H, G, P, N, R, K = 1, 4, 2, 1, 2, 4, 2, 1
    sp = lambda v: np.log1p(np.exp(v))
    bc = (Bt, T, G, R, N) if mimo else (Bt, T, G, N)
    arrs = [rng.standard_normal((Bt, T, H, P)), sp(rng.standard_normal((Bt, T, H)) - 1.0),
            -np.exp(rng.uniform(0, 1, H)), 1 / (1 + np.exp(-rng.standard_normal((Bt, T, H)))),
            rng.uniform(-1, 1, (Bt, T, H, K)), rng.standard_normal(bc) / 2, rng.standard_normal(bc) / 2,
            rng.standard_normal(H)]
    W = [1 + 0.3 * rng.standard_normal((H, R, P)), 1 + 0.3 * rng.standard_normal((H, R, P))] if mimo else [None, None]
    st = [0.5 * rng.standard_normal((Bt, H, N, P)), 0.3 * rng.standard_normal((Bt, H, N, P)),
          rng.uniform(-2, 2, (Bt, H, K))]
    ts = [T64(a).requires_grad_() for a in arrs]
    ws = [None if w is None else T64(w).requires_grad_() for w in W]
    ss = [T64(a).requires_grad_() for a in st]
    fn = lambda *a: ag.Mamba3Scan.apply(*a, 4)
    assert torch.autograd.gradcheck(fn, (*ts, *ws, *ss), eps=1e-6, atol=1e-6, rtol=1e-5)


def test_siso_rejects_rank_vectors():
    x = torch.zeros(1, 2, 1, 2, dtype=torch.float64)
    B = torch.zeros(1, 2, 1, 4, dtype=torch.float64)
    with pytest.raises(ValueError):
        ag.mamba3_scan(x, torch.zeros(1, 2, 1), torch.zeros(1), torch.zeros(1, 2, 1), torch.zeros(1, 2, 1, 2),
                       B, B, torch.zeros(1), W_x=torch.ones(1, 1, 2))
