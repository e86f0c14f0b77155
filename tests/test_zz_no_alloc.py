"""m3_siso_chunked_fwd_noalloc: the SISO chunked forward for callers that
cannot allocate device memory (a plugin inside a framework that owns all
device memory, or a host that must not allocate while serving).  Its scratch
is a buffer built into the library instead of a caller-provided workspace.

Checked through the C ABI against m3_siso_chunked_fwd on the same inputs, on
two calls in a row (the buffer keeps the first call's contents when the
second one runs).  This file is collected last on purpose."""
import ctypes

import pytest
import torch

from helpers import TOL, relerr
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3

pytestmark = pytest.mark.gpu

_VP = ctypes.c_void_p
SCRATCH_BYTES = 32 * 1024 * 1024        # M3_NOALLOC_SCRATCH_BYTES in include/m3.h


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
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


def test_noalloc_matches_the_workspace_entry_point_on_two_calls():
    L = _lib()
    # a long sequence over few (b, h) lanes: the segmented path, which needs scratch
    Bt, T, H, P, N = 1, 3000, 2, 64, 128
    dims = m3.Dims(Bt, T, H, P, N, 1, 64)
    need = m3.workspace_bytes(m3.M3_WS_SISO, dims, m3.M3_BF16)
    assert 0 < need <= SCRATCH_BYTES
    for seed in (401, 402):
        inp = gen.scan_inputs(Bt, T, H, P, N, dtype="bf16", seed=seed, dt_shift=-4.0)
        d = {k: v.cuda() for k, v in inp.items() if isinstance(v, torch.Tensor)}
        ref = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"], 64)
        out = (torch.empty_like(d["x"]), torch.empty(Bt, H, N, P, device="cuda"),
               torch.empty(Bt, H, N, P, device="cuda"), torch.empty(Bt, H, N // 2, device="cuda"))
        assert _noalloc(L, d, dims, out) == m3.M3_OK
        torch.cuda.synchronize()
        for got, want in zip(out, ref):
            assert relerr(got, want) <= TOL[torch.bfloat16]
        assert m3.device_error() == m3.M3_OK


def test_noalloc_scratch_need_fits_its_buffer():
    _lib()
    # the segment plan caps the number of segment slots, so the scratch need
    # stays below the built-in buffer for any sequence length
    for lanes in (1, 2, 7, 32, 63, 95):
        for T in (4096, 32768, 1 << 20, 1 << 24):
            dims = m3.Dims(1, T, lanes, 64, 128, 1, 64)
            assert m3.workspace_bytes(m3.M3_WS_SISO, dims, m3.M3_BF16) <= SCRATCH_BYTES
