"""m3_siso_chunked_fwd_noalloc: the SISO chunked forward for callers that
cannot allocate device memory (a plugin inside a framework that owns all
device memory, or a host that must not allocate while serving).  Its scratch
is a buffer built into the library instead of a caller-provided workspace.

Checked through the C ABI on two calls in a row (the buffer keeps the first
call's contents when the second one runs): bit for bit against
m3_siso_chunked_fwd on the same inputs, since both run the same deterministic
kernels, and against the fp64 oracle within the bf16 bar.  This file is
collected last on purpose."""
import ctypes
import os
import re

import pytest
import torch

import oracle
from helpers import TOL, relerr
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.inputs import to_f64

pytestmark = pytest.mark.gpu

_VP = ctypes.c_void_p
_HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "m3.h")


def _scratch_bytes():
    """M3_NOALLOC_SCRATCH_BYTES as include/m3.h defines it."""
    m = re.search(r"#define\s+M3_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\s*\*\s*(\d+)u\)", open(_HEADER).read())
    assert m, "M3_NOALLOC_SCRATCH_BYTES not found in include/m3.h"
    return int(m.group(1)) * int(m.group(2)) * int(m.group(3))


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
    oracle.build_oracle()
    L = m3.lib()
    fn = L.m3_siso_chunked_fwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int, ctypes.POINTER(m3.BcNorm), _VP, _VP,
                   _VP, m3.Dims, _VP, _VP, _VP, _VP, _VP]
    return L


def _noalloc(L, d, dims, out):
    p = lambda t: None if t is None else t.data_ptr()
    y, hf, uf, af = out
    stream = torch.cuda.current_stream().cuda_stream
    return L.m3_siso_chunked_fwd_noalloc(p(d["x"]), p(d["dt"]), p(d["A"]), p(d["lam"]), p(d["theta"]), p(d["B"]),
                                         p(d["C"]), p(d["D"]), m3.M3_BF16, None, None, None, None, dims, p(y),
                                         p(hf), p(uf), p(af), stream)


def test_noalloc_matches_the_workspace_entry_point_and_the_oracle_on_two_calls():
    L = _lib()
    # a long sequence over few (b, h) lanes: the segmented path, which needs scratch
    Bt, T, H, P, N = 1, 3000, 2, 64, 128
    dims = m3.Dims(Bt, T, H, P, N, 1, 64)
    need = m3.workspace_bytes(m3.M3_WS_SISO, dims, m3.M3_BF16)
    assert 0 < need <= _scratch_bytes()
    for seed in (401, 402):
        inp = gen.scan_inputs(Bt, T, H, P, N, dtype="bf16", seed=seed, dt_shift=-4.0)
        d = {k: v.cuda() for k, v in inp.items() if isinstance(v, torch.Tensor)}
        ref = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"], 64)
        out = (torch.full_like(d["x"], float("nan")), torch.full((Bt, H, N, P), float("nan"), device="cuda"),
               torch.full((Bt, H, N, P), float("nan"), device="cuda"),
               torch.full((Bt, H, N // 2), float("nan"), device="cuda"))
        assert _noalloc(L, d, dims, out) == m3.M3_OK
        torch.cuda.synchronize()
        assert m3.device_error() == m3.M3_OK
        for got, want in zip(out, ref):
            assert torch.equal(got, want)
        orc = oracle.siso_loop(*(to_f64(inp[k]) for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")))
        for got, want in zip(out, orc):
            assert relerr(got, want) <= TOL[torch.bfloat16]


def test_noalloc_scratch_need_fits_its_buffer():
    _lib()
    # the segment plan caps the number of segment slots, so the scratch need
    # stays below the built-in buffer for any sequence length
    cap = _scratch_bytes()
    for lanes in (1, 2, 7, 32, 63, 95):
        for T in (4096, 32768, 1 << 20, 1 << 24):
            dims = m3.Dims(1, T, lanes, 64, 128, 1, 64)
            assert m3.workspace_bytes(m3.M3_WS_SISO, dims, m3.M3_BF16) <= cap
