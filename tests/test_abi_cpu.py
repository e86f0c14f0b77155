"""The C-ABI library: it loads, exports every symbol include/m3.h declares, and
rejects bad arguments on the host before any launch (CPU only: no call here
passes validation, so no kernel is ever enqueued)."""
import ctypes
import os
import re

import pytest

from state_space_lm_b200 import build as m3build
from state_space_lm_b200 import m3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    m3build.build()
    return m3.lib()


def header_symbols():
    src = open(os.path.join(ROOT, "include", "m3.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(m3_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    syms = header_symbols()
    assert len(syms) >= 9
    for s in syms:
        assert hasattr(L, s), s
    assert set(syms) == set(m3.ABI_FUNCTIONS)


def test_status_strings_and_limits(L):
    for code in range(6):
        s = m3.status_string(code)
        assert s.startswith("M3_")
    assert "unknown" in m3.status_string(99)
    lim = m3.limits()
    assert lim["max_dstate"] >= 128 and lim["max_headdim"] >= 64 and lim["max_rank"] >= 4


FAKE = 0x10000      # aligned, never dereferenced: every call below fails validation
MIS = 0x10004       # misaligned


def dims(**kw):
    base = dict(batch=2, seqlen=8, nheads=2, headdim=4, dstate=4, rank=1, chunk=4, ngroups=0, rope_pairs=0)
    base.update(kw)
    return m3.Dims(*[base[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate", "rank", "chunk",
                                       "ngroups", "rope_pairs")])


def siso(L, d, x=FAKE, dt=FAKE, A=FAKE, lam=FAKE, theta=FAKE, B=FAKE, C=FAKE, D=FAKE, dtype=m3.M3_BF16,
         y=FAKE, ws=None, nbytes=0):
    return L.m3_siso_chunked_fwd(x, dt, A, lam, theta, B, C, D, dtype, None, None, None, None, d, y,
                                 None, None, None, ws, nbytes, None)


def test_siso_validation(L):
    assert siso(L, dims(dstate=5)) == m3.M3_ERR_INVALID_ARG              # odd N: RoPE needs pairs
    assert siso(L, dims(dstate=0)) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(nheads=0)) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(batch=-1)) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(seqlen=-3)) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(chunk=0)) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(), x=None) == m3.M3_ERR_INVALID_ARG              # null required pointer
    assert siso(L, dims(), theta=None) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(), y=MIS) == m3.M3_ERR_INVALID_ARG               # misaligned
    assert siso(L, dims(), dtype=7) == m3.M3_ERR_INVALID_ARG
    assert siso(L, dims(dstate=512)) == m3.M3_ERR_UNSUPPORTED
    assert siso(L, dims(headdim=512)) == m3.M3_ERR_UNSUPPORTED
    assert siso(L, dims(dstate=256, headdim=128)) == m3.M3_ERR_UNSUPPORTED
    # an empty batch is valid and enqueues nothing
    n0 = m3.launch_count()
    assert siso(L, dims(batch=0), x=None, dt=None, lam=None, theta=None, B=None, C=None, y=None) == m3.M3_OK
    assert m3.launch_count() == n0


def test_mimo_validation(L):
    def mimo(d, **kw):
        a = dict(x=FAKE, dt=FAKE, A=FAKE, lam=FAKE, theta=FAKE, B=FAKE, C=FAKE, D=FAKE, Wx=None, Wy=None)
        a.update(kw)
        return L.m3_mimo_chunked_fwd(a["x"], a["dt"], a["A"], a["lam"], a["theta"], a["B"], a["C"], a["D"],
                                     a["Wx"], a["Wy"], m3.M3_BF16, None, None, None, None, d, FAKE, None,
                                     None, None, None, 0, None)
    assert mimo(dims(rank=0)) == m3.M3_ERR_INVALID_ARG
    assert mimo(dims(rank=64)) == m3.M3_ERR_UNSUPPORTED
    assert mimo(dims(rank=2), Wx=MIS) == m3.M3_ERR_INVALID_ARG


def test_norm_validation(L):
    nrm = m3.BcNorm(FAKE, FAKE, None, None, -1.0)                       # negative eps
    rc = L.m3_siso_chunked_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16,
                               ctypes.byref(nrm), None, None, None, dims(), FAKE, None, None, None, None,
                               0, None)
    assert rc == m3.M3_ERR_INVALID_ARG
    nrm = m3.BcNorm(MIS, None, None, None, 1e-5)
    rc = L.m3_siso_chunked_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16,
                               ctypes.byref(nrm), None, None, None, dims(), FAKE, None, None, None, None,
                               0, None)
    assert rc == m3.M3_ERR_INVALID_ARG


def test_decode_rope_discretize_validation(L):
    d = dims()
    assert L.m3_step_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16, None, dims(dstate=3),
                            FAKE, FAKE, FAKE, FAKE, None) == m3.M3_ERR_INVALID_ARG
    assert L.m3_step_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16, None, d,
                            None, FAKE, FAKE, FAKE, None) == m3.M3_ERR_INVALID_ARG
    assert L.m3_rope_bc(FAKE, FAKE, m3.M3_BF16, FAKE, FAKE, None, None, dims(dstate=7), FAKE, FAKE, None,
                        None) == m3.M3_ERR_INVALID_ARG
    assert L.m3_rope_bc(FAKE, None, m3.M3_BF16, FAKE, FAKE, None, None, d, FAKE, FAKE, None,
                        None) == m3.M3_ERR_INVALID_ARG
    assert L.m3_discretize(FAKE, None, FAKE, d, FAKE, FAKE, FAKE, None) == m3.M3_ERR_INVALID_ARG
    assert L.m3_discretize(FAKE, FAKE, FAKE, dims(nheads=0), FAKE, FAKE, FAKE, None) == m3.M3_ERR_INVALID_ARG


def test_rank_decode_validation(L):
    def full(d, Wx=None, h=FAKE, u=FAKE, dtype=m3.M3_BF16):
        return L.m3_mimo_step_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, Wx, None, dtype, None, d,
                                     h, u, FAKE, FAKE, None)

    def fact(d, bp=FAKE, xp=FAKE, Wy=None):
        return L.m3_step_decode_factored(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, Wy, m3.M3_BF16,
                                         None, d, FAKE, bp, xp, FAKE, FAKE, None)

    assert full(dims(rank=0)) == m3.M3_ERR_INVALID_ARG
    assert full(dims(rank=9)) == m3.M3_ERR_UNSUPPORTED
    assert full(dims(rank=2, headdim=6)) == m3.M3_ERR_UNSUPPORTED     # rows are streamed 4-wide
    assert full(dims(rank=2), Wx=MIS) == m3.M3_ERR_INVALID_ARG
    assert full(dims(rank=2), u=None) == m3.M3_ERR_INVALID_ARG         # the full state needs prev_Bx
    assert full(dims(rank=2), h=MIS) == m3.M3_ERR_INVALID_ARG
    assert full(dims(rank=2), dtype=5) == m3.M3_ERR_INVALID_ARG
    assert fact(dims(dstate=5)) == m3.M3_ERR_INVALID_ARG
    assert fact(dims(rank=1), bp=None) == m3.M3_ERR_INVALID_ARG        # the factored state needs b_prev
    assert fact(dims(rank=3), xp=MIS) == m3.M3_ERR_INVALID_ARG
    assert fact(dims(rank=3), Wy=MIS) == m3.M3_ERR_INVALID_ARG


def test_groups_and_rope_pairs_validation(L):
    """B/C groups must divide the heads; rotated pairs are 1..dstate/2; 0 means
    the default (one group per head, every pair)."""
    def rope(d):
        return L.m3_rope_bc(FAKE, FAKE, m3.M3_BF16, FAKE, FAKE, None, None, d, FAKE, FAKE, None, None)

    def step(d):
        return L.m3_step_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16, None, d,
                                FAKE, FAKE, FAKE, FAKE, None)

    def fact(d):
        return L.m3_step_decode_factored(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, m3.M3_BF16,
                                         None, d, FAKE, FAKE, FAKE, FAKE, FAKE, None)

    base = dict(nheads=6, dstate=8)
    for bad in (dict(ngroups=4), dict(ngroups=-1), dict(rope_pairs=5), dict(rope_pairs=-2)):
        d = dims(**base, **bad)
        assert siso(L, d) == m3.M3_ERR_INVALID_ARG, bad
        assert rope(d) == m3.M3_ERR_INVALID_ARG, bad
        assert step(d) == m3.M3_ERR_INVALID_ARG, bad
        assert fact(d) == m3.M3_ERR_INVALID_ARG, bad
    # valid groups and pairs get past the size checks (a null x then fails)
    for ok in (dict(ngroups=1), dict(ngroups=3), dict(ngroups=6, rope_pairs=1), dict(rope_pairs=4)):
        assert siso(L, dims(**base, **ok), x=None) == m3.M3_ERR_INVALID_ARG
        assert m3.workspace_bytes(m3.M3_WS_SISO, dims(**base, **ok), m3.M3_BF16) == 0
    long3 = dict(batch=1, seqlen=32768, nheads=32, headdim=64, dstate=128, chunk=128)
    assert m3.workspace_bytes(m3.M3_WS_SISO, dims(**long3, ngroups=1, rope_pairs=32), m3.M3_BF16) > 0
    # a pair count that is not a multiple of 4 runs on the FFMA path: no scratch
    assert m3.workspace_bytes(m3.M3_WS_SISO, dims(**long3, ngroups=1, rope_pairs=30), m3.M3_BF16) == 0
    assert m3.workspace_bytes(m3.M3_WS_SISO, dims(**long3, ngroups=5), m3.M3_BF16) == 0


def test_backward_validation(L):
    """m3_chunked_bwd rejects bad arguments before any launch."""
    g = m3.Grads(*([None] * len(m3.GRAD_FIELDS)))

    def bwd(d, dy=FAKE, grads=True, ws=None, nbytes=0, dtype=m3.M3_BF16, gx=None):
        gg = m3.Grads(*([gx] + [None] * (len(m3.GRAD_FIELDS) - 1))) if gx is not None else g
        return L.m3_chunked_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, dtype, None, None,
                                None, None, d, dy, None, None, None, ctypes.byref(gg) if grads else None, ws,
                                nbytes, None)

    assert bwd(dims(), grads=False) == m3.M3_ERR_INVALID_ARG           # no gradient struct
    assert bwd(dims(), dy=None) == m3.M3_ERR_INVALID_ARG               # dy is required
    assert bwd(dims(dstate=5)) == m3.M3_ERR_INVALID_ARG
    assert bwd(dims(chunk=0)) == m3.M3_ERR_INVALID_ARG
    assert bwd(dims(rank=9)) == m3.M3_ERR_UNSUPPORTED
    assert bwd(dims(), dtype=7) == m3.M3_ERR_INVALID_ARG
    assert bwd(dims(nheads=6, ngroups=4)) == m3.M3_ERR_INVALID_ARG      # groups must divide the heads
    assert bwd(dims(), gx=MIS) == m3.M3_ERR_INVALID_ARG                 # misaligned gradient buffer
    # the workspace is required and checked before any launch
    need = m3.workspace_bytes(m3.M3_WS_BWD_SISO, dims(), m3.M3_BF16)
    assert need > 0
    assert bwd(dims()) == m3.M3_ERR_WORKSPACE
    assert bwd(dims(), ws=FAKE, nbytes=need - 16) == m3.M3_ERR_WORKSPACE
    # workspace grows with the sequence (one entering state per chunk)
    assert m3.workspace_bytes(m3.M3_WS_BWD_SISO, dims(seqlen=64), m3.M3_BF16) > need


def test_workspace_query(L):
    for which in (m3.M3_WS_SISO, m3.M3_WS_MIMO):
        n = m3.workspace_bytes(which, dims(), m3.M3_BF16)
        assert n >= 0
    # long sequences over few lanes need scratch for the segment states
    long3 = dims(batch=1, seqlen=32768, nheads=32, headdim=64, dstate=128, chunk=128)
    need = m3.workspace_bytes(m3.M3_WS_SISO, long3, m3.M3_BF16)
    assert need > 0
    assert m3.workspace_bytes(m3.M3_WS_SISO, long3, m3.M3_F32) == 0      # FFMA path: no scratch
    many = dims(batch=8, seqlen=2048, nheads=16, headdim=64, dstate=128, chunk=64)
    assert m3.workspace_bytes(m3.M3_WS_SISO, many, m3.M3_BF16) == 0      # enough lanes: one segment
    # a missing or short workspace is rejected before any launch
    assert siso(L, long3) == m3.M3_ERR_WORKSPACE
    assert siso(L, long3, ws=FAKE, nbytes=need - 16) == m3.M3_ERR_WORKSPACE
    # a chunk request past 2^30 behaves as 2^30: the same path and scratch as
    # any other multiple of the kernel's 64-row chunk
    for huge in (1 << 30, (1 << 31) + 128, (1 << 32) + 128, (1 << 62)):
        big = dims(batch=1, seqlen=32768, nheads=32, headdim=64, dstate=128, chunk=huge)
        assert m3.workspace_bytes(m3.M3_WS_SISO, big, m3.M3_BF16) == need, huge
        assert siso(L, big) == m3.M3_ERR_WORKSPACE, huge


def test_sizes_past_the_index_limits(L):
    """Lane counts past a 1-D grid and tensors past 2^46 elements are
    M3_ERR_UNSUPPORTED at every entry point, before any launch, with no
    integer overflow in the checks themselves."""
    g = m3.Grads(*([None] * len(m3.GRAD_FIELDS)))
    lanes = dict(batch=1 << 24, nheads=256)                             # 2^32 lanes
    elems = dict(batch=1 << 20, seqlen=1 << 30, nheads=16, headdim=64, dstate=128)   # 2^61 elements
    wrap = dict(batch=1 << 24, seqlen=1 << 31, nheads=4096, headdim=256, dstate=256)  # 2^75: wraps int64
    for kw in (lanes, elems, wrap):
        d = dims(**kw)
        assert siso(L, d) == m3.M3_ERR_UNSUPPORTED, kw
        assert L.m3_rope_bc(FAKE, FAKE, m3.M3_BF16, FAKE, FAKE, None, None, d, FAKE, FAKE, None,
                            None) == m3.M3_ERR_UNSUPPORTED, kw
        assert L.m3_chunked_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, m3.M3_BF16, None,
                                None, None, None, d, FAKE, None, None, None, ctypes.byref(g), None, 0,
                                None) == m3.M3_ERR_UNSUPPORTED, kw
        assert m3.workspace_bytes(m3.M3_WS_BWD_SISO, d, m3.M3_BF16) == 0, kw
    d = dims(**lanes)
    assert L.m3_step_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16, None, d,
                            FAKE, FAKE, FAKE, FAKE, None) == m3.M3_ERR_UNSUPPORTED
    for big in (dims(batch=1 << 40, seqlen=1 << 40), dims(batch=1 << 30, seqlen=1 << 17, nheads=1 << 20)):
        assert L.m3_discretize(FAKE, FAKE, FAKE, big, FAKE, FAKE, FAKE, None) == m3.M3_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """Without the built CUDA library every call raises: there is no other
    implementation behind the binding's names."""
    import importlib
    mod = importlib.reload(m3)
    monkeypatch.setattr(mod, "LIB", str(tmp_path / "nonexistent_libm3.so"))
    monkeypatch.setattr(mod, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mod.lib()
    with pytest.raises(RuntimeError):
        mod.limits()
    importlib.reload(m3)


def test_injected_launch_failure(L):
    """m3_debug_fail_next_launches: calls that pass their checks report
    M3_ERR_CUDA and launch nothing; calls that fail their checks keep their
    own status and do not use up the count."""
    L = m3.lib()        # this module's current binding (another test reloads it)
    n0 = m3.launch_count()
    g = m3.Grads(*([None] * len(m3.GRAD_FIELDS)))
    d = dims()
    need = m3.workspace_bytes(m3.M3_WS_BWD_SISO, d, m3.M3_BF16)
    valid = [
        lambda: siso(L, d),
        lambda: L.m3_mimo_chunked_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, m3.M3_BF16, None,
                                      None, None, None, dims(rank=2), FAKE, None, None, None, None, 0, None),
        lambda: L.m3_rope_bc(FAKE, FAKE, m3.M3_BF16, FAKE, FAKE, None, None, d, FAKE, FAKE, None, None),
        lambda: L.m3_discretize(FAKE, FAKE, FAKE, d, FAKE, FAKE, FAKE, None),
        lambda: L.m3_step_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, m3.M3_BF16, None, d, FAKE, FAKE,
                                 FAKE, FAKE, None),
        lambda: L.m3_step_decode_factored(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, m3.M3_BF16,
                                          None, dims(rank=2), FAKE, FAKE, FAKE, FAKE, FAKE, None),
        lambda: L.m3_chunked_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, m3.M3_BF16, None, None,
                                 None, None, d, FAKE, None, None, None, ctypes.byref(g), FAKE, need, None),
    ]
    try:
        m3.debug_fail_next_launches(len(valid))
        assert siso(L, dims(dstate=5)) == m3.M3_ERR_INVALID_ARG      # a failed check does not count
        for call in valid:
            assert call() == m3.M3_ERR_CUDA
        # the count is used up; another failed check still reports itself
        assert siso(L, dims(headdim=512)) == m3.M3_ERR_UNSUPPORTED
        assert m3.launch_count() == n0                                # nothing was enqueued
    finally:
        m3.debug_fail_next_launches(0)
