"""The timeout path of the bounded waits, exercised on the GPU without a
fault, and the host-side launch-failure hook (marked gpu).

Every wait inside the tensor-core kernels is bounded (about one second);
when one runs out the kernel records the wait site in a device error word
and returns normally, and m3_device_error reports M3_ERR_TIMEOUT.  The
self-test kernel waits, with the same bounded wait, on a barrier that
nothing ever completes, so the wait runs out for certain; the context must
stay usable afterwards.
"""
import time

import pytest
import torch

import oracle
from helpers import relerr
from state_space_lm_b200 import inputs as gen
from state_space_lm_b200 import m3
from state_space_lm_b200.inputs import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from state_space_lm_b200 import build
    build.build()
    oracle.build_oracle()


def test_bounded_wait_runs_out_and_the_context_survives():
    assert m3.device_error() == m3.M3_OK          # nothing pending
    t0 = time.perf_counter()
    m3.selftest_bounded_wait()
    status, site = m3.device_error(with_site=True)
    waited = time.perf_counter() - t0
    assert status == m3.M3_ERR_TIMEOUT and site == m3.M3_SELFTEST_SITE
    assert 0.2 < waited < 30.0, waited
    assert m3.device_error() == m3.M3_OK          # the report clears the word
    # the same process and context still compute correctly
    inp = gen.scan_inputs(2, 130, 2, 64, 128, dtype="bf16", seed=700)
    d = {k: v.cuda() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    keys = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
    y, hf, uf, af = m3.siso_chunked_fwd(*[d[k] for k in keys], 64)
    torch.cuda.synchronize()
    ref = oracle.siso_loop(**{k: to_f64(inp[k]) for k in keys})
    assert max(relerr(g, r) for g, r in zip((y, hf, uf, af), ref)) <= 2e-2
    assert m3.device_error() == m3.M3_OK


def test_injected_launch_failure_raises_and_enqueues_nothing():
    """The host-side failure hook: the binding raises M3Error(M3_ERR_CUDA),
    the outputs keep their contents, and the next call computes normally."""
    inp = gen.scan_inputs(1, 20, 2, 8, 8, dtype="f32", seed=41)
    d = {k: v.cuda() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    keys = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
    out = (torch.full((1, 20, 2, 8), -7.0, device="cuda"), torch.full((1, 2, 8, 8), -7.0, device="cuda"),
           torch.full((1, 2, 8, 8), -7.0, device="cuda"), torch.full((1, 2, 4), -7.0, device="cuda"))
    n0 = m3.launch_count()
    m3.debug_fail_next_launches(1)
    try:
        with pytest.raises(m3.M3Error) as err:
            m3.siso_chunked_fwd(*[d[k] for k in keys], 4, out=out)
        assert err.value.status == m3.M3_ERR_CUDA
    finally:
        m3.debug_fail_next_launches(0)
    torch.cuda.synchronize()
    assert m3.launch_count() == n0
    assert all(bool((o == -7.0).all()) for o in out)
    y, hf, uf, af = m3.siso_chunked_fwd(*[d[k] for k in keys], 4, out=out)
    torch.cuda.synchronize()
    ref = oracle.siso_loop(**{k: to_f64(inp[k]) for k in keys})
    assert max(relerr(g, r) for g, r in zip((y, hf, uf, af), ref)) <= 1e-5
