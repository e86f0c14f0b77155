"""Shared helpers of the parity tests: error metric, lane sampling, canaries."""
import os

import numpy as np
import torch

from state_space_lm_b200.inputs import to_f64

# Accuracy bars (max relative error, normwise per output tensor): 1e-5 for
# fp32 inputs; 2e-2 for bf16 inputs with fp32 accumulation and state.
TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


# Every relerr() call also records the per-element metric
# |g - o| / (|o| + 1e-3 max|o|) (the survey's second reported figure) with the
# normwise one, keyed by the running test; conftest prints the worst of each
# at the end of the session and, when M3_ERRLOG names a file, writes them all.
ERR_LOG = []


def elemerr(got, ref):
    """max_i |g_i - o_i| / (|o_i| + 1e-3 max_j |o_j|) (per-element relative)."""
    g = got if isinstance(got, np.ndarray) else to_f64(got)
    o = ref if isinstance(ref, np.ndarray) else to_f64(ref)
    assert g.shape == o.shape, (g.shape, o.shape)
    if not o.size:
        return 0.0
    floor = 1e-3 * np.max(np.abs(o))
    if floor == 0.0:
        return float(np.max(np.abs(g)))
    return float(np.max(np.abs(g - o) / (np.abs(o) + floor)))


def relerr(got, ref):
    """max_i |g - o| / max_i |o| (normwise max-relative; robust near zeros)."""
    g = got if isinstance(got, np.ndarray) else to_f64(got)
    o = ref if isinstance(ref, np.ndarray) else to_f64(ref)
    assert g.shape == o.shape, (g.shape, o.shape)
    den = np.max(np.abs(o)) if o.size else 0.0
    if den == 0.0:
        r = float(np.max(np.abs(g))) if g.size else 0.0
    else:
        r = float(np.max(np.abs(g - o)) / den)
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    ERR_LOG.append((test, tuple(o.shape), r, elemerr(g, o)))
    return r


def cuda(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def f64(d, keys):
    return {k: (to_f64(d[k]) if d.get(k) is not None else None) for k in keys}


SCAN_KEYS = ("x", "dt", "A", "lam", "theta", "B", "C", "D")


def lane_inputs(inp, b, h):
    """Slice one (b, h) lane out of full-size scan inputs, widened to float64."""
    out = {}
    for k in SCAN_KEYS:
        v = inp[k]
        if k in ("A", "D"):
            out[k] = to_f64(v[h:h + 1])
        else:
            out[k] = to_f64(v[b:b + 1, :, h:h + 1])
    for k in ("Wx", "Wy"):
        if inp.get(k) is not None:
            out[k] = to_f64(inp[k][h:h + 1])
    return out


def norm_f64(inp, h=None):
    if "normw_B" not in inp:
        return None
    d = {k: to_f64(inp[k]) for k in ("normw_B", "normw_C", "bias_B", "bias_C")}
    if h is not None:
        d["bias_B"] = d["bias_B"][h:h + 1]
        d["bias_C"] = d["bias_C"][h:h + 1]
    d["eps"] = inp["eps"]
    return d


def norm_dev(inp):
    if "normw_B" not in inp:
        return None
    return {k: inp[k].cuda() for k in ("normw_B", "normw_C", "bias_B", "bias_C")} | {"eps": inp["eps"]}


def sample_lanes(Bt, H):
    lanes = {(0, 0), (Bt - 1, H - 1), (Bt // 2, H // 3)}
    return sorted(lanes)


class Canary:
    """A device buffer with sentinel padding on both sides of the view handed
    to the library; ``check()`` asserts nothing was written outside it."""

    PAD = 256

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.buf = torch.full((n + 2 * self.PAD,), -12345.0, dtype=dtype, device="cuda")
        self.t = self.buf[self.PAD:self.PAD + n].view(*shape)

    def check(self):
        lo = self.buf[:self.PAD]
        hi = self.buf[-self.PAD:]
        assert bool((lo == -12345.0).all()) and bool((hi == -12345.0).all()), "write outside the output"
