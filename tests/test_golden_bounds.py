"""The pages' printed accuracy figures as golden bounds (fixtures in
tests/golden/pages_printed_bounds.json, each with its source).

CPU: the fp64 oracle run as the pages' split schedules (a prefill by the loop,
then the rest token by token on the carried state) against the one-shot
loop, on the printed MIMO shape; the drift must stay within the printed
bounds.  GPU (marked): the fp32 chunked forward against a prefill of 9
tokens plus 8 decode steps on the printed B=2, L=17 shape, within the
printed fp32 tolerances.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_printed_bounds.json")))


def _mimo_inputs(rng, Bt, T, H, P, N, R):
    sp = lambda v: np.log1p(np.exp(v))
    return dict(
        x=rng.standard_normal((Bt, T, H, P)), dt=sp(rng.standard_normal((Bt, T, H)) - 1.0),
        A=-np.exp(rng.uniform(0, 1, H)), lam=1 / (1 + np.exp(-rng.standard_normal((Bt, T, H)))),
        theta=rng.uniform(-np.pi / 8, np.pi / 8, (Bt, T, H, N // 2)),
        B=rng.standard_normal((Bt, T, H, R, N)) / np.sqrt(N), C=rng.standard_normal((Bt, T, H, R, N)) / np.sqrt(N),
        D=rng.standard_normal(H)), 1 + 0.02 * rng.standard_normal((H, R, P)), 1 + 0.02 * rng.standard_normal((H, R, P))


def test_mimo_split_drift_within_printed_bound():
    g = GOLD["mimo_split_drift"]
    R, T, H, P, N = g["rank"], g["seqlen"], g["nheads"], g["headdim"], g["dstate"]
    inp, Wx, Wy = _mimo_inputs(np.random.default_rng(900), 1, T, H, P, N, R)
    y1, h1, u1, a1 = oracle.mimo_loop(**inp, Wx=Wx, Wy=Wy)
    worst_y = worst_h = 0.0
    for sched in g["schedules"]:
        assert sum(sched) == T
        ys, h, u, a, t0 = [], None, None, None, 0
        for n in sched:
            piece = {k: (v[:, t0:t0 + n] if k in ("x", "dt", "lam", "theta", "B", "C") else v) for k, v in inp.items()}
            y, h, u, a = oracle.mimo_loop(**piece, Wx=Wx, Wy=Wy, h0=h, prevBx0=u, angle0=a)
            ys.append(y)
            t0 += n
        worst_y = max(worst_y, float(np.max(np.abs(np.concatenate(ys, 1) - y1))))
        worst_h = max(worst_h, float(np.max(np.abs(h - h1))))
    assert worst_y <= g["y_max_abs"], worst_y
    assert worst_h <= g["state_max_abs"], worst_h


@pytest.mark.gpu
@pytest.mark.parametrize("rank", [1, 3])
def test_fp32_forward_vs_prefill_steps_within_printed_tolerance(rank):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    from state_space_lm_b200 import inputs as gen
    from state_space_lm_b200 import m3
    build.build()
    g = GOLD["forward_vs_prefill_step"]
    Bt, T, k = g["batch"], g["seqlen"], g["prefix"]
    H, P, N = 4, 8, 16
    inp = gen.scan_inputs(Bt, T, H, P, N, rank=rank, dtype="f32", seed=901 + rank, mimo_weights=rank > 1)
    d = {kk: v.cuda() for kk, v in inp.items() if isinstance(v, torch.Tensor)}
    keys = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
    mimo = rank > 1
    kw = dict(W_x=d["Wx"], W_y=d["Wy"]) if mimo else {}
    fwd = m3.mimo_chunked_fwd if mimo else m3.siso_chunked_fwd
    y_full = fwd(*[d[kk] for kk in keys], 8, **kw)[0]
    pre = {kk: (v[:, :k].contiguous() if kk in ("x", "dt", "lam", "theta", "B", "C") else v) for kk, v in d.items()}
    _, h, u, a = fwd(*[pre[kk] for kk in keys], 8, **kw)
    ys = []
    for t in range(k, T):
        args = [d[kk][:, t].contiguous() if kk in ("x", "dt", "lam", "theta", "B", "C") else d[kk] for kk in keys]
        if mimo:
            ys.append(m3.mimo_step_decode(*args, h, u, a, **kw))
        else:
            ys.append(m3.step_decode(*args, h, u, a))
    torch.cuda.synchronize()
    got, ref = torch.stack(ys, 1), y_full[:, k:]
    err = (got - ref).abs()
    assert float(err.max()) <= g["fp32_atol"] + g["fp32_rtol"] * float(ref.abs().max()), float(err.max())
