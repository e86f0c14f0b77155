"""Python binding of the C ABI in ``include/m3.h`` (ctypes).

Argument marshalling only: every step of the scan runs in the CUDA library.
Tensors are torch CUDA tensors (PyTorch supplies device memory and streams);
outputs that the caller does not pass are allocated with ``torch.empty``.
If the library has not been built, every call raises ``RuntimeError`` -- there
is no other implementation behind these names.
"""
import ctypes
import os

import torch

from .build import LIB

M3_OK, M3_ERR_INVALID_ARG, M3_ERR_UNSUPPORTED, M3_ERR_WORKSPACE, M3_ERR_CUDA, M3_ERR_TIMEOUT = range(6)
M3_F32, M3_BF16 = 0, 1
M3_WS_SISO, M3_WS_MIMO, M3_WS_BWD_SISO, M3_WS_BWD_MIMO = 0, 1, 2, 3

_DTYPE = {torch.float32: M3_F32, torch.bfloat16: M3_BF16}

ABI_FUNCTIONS = (
    "m3_get_limits", "m3_discretize", "m3_rope_bc", "m3_siso_chunked_fwd",
    "m3_mimo_chunked_fwd", "m3_step_decode", "m3_workspace_bytes", "m3_status_string",
    "m3_launch_count", "m3_device_error", "m3_siso_chunked_fwd_noalloc", "m3_mimo_step_decode",
    "m3_step_decode_factored", "m3_chunked_bwd", "m3_selftest_bounded_wait", "m3_debug_fail_next_launches",
)
M3_SELFTEST_SITE = 99

GRAD_FIELDS = ("dx", "ddt", "dA", "dlam", "dtheta", "dB", "dC", "dD", "dW_x", "dW_y",
               "dnormw_B", "dnormw_C", "dbias_B", "dbias_C", "dh0", "dprevBx0", "dangle0")


class M3Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s" % (where, status_string(status)))


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("rank", ctypes.c_int64),
                ("chunk", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("rope_pairs", ctypes.c_int64)]


class BcNorm(ctypes.Structure):
    _fields_ = [("normw_B", ctypes.c_void_p), ("normw_C", ctypes.c_void_p),
                ("bias_B", ctypes.c_void_p), ("bias_C", ctypes.c_void_p),
                ("eps", ctypes.c_float)]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_FIELDS]


class Limits(ctypes.Structure):
    _fields_ = [("max_dstate", ctypes.c_int64), ("max_headdim", ctypes.c_int64),
                ("max_state_elems", ctypes.c_int64), ("max_rank", ctypes.c_int64)]


_lib = None
_VP = ctypes.c_void_p


def library_path():
    return LIB


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise RuntimeError("the CUDA library %s is missing: run `python -m state_space_lm_b200.build`"
                           % LIB)
    L = ctypes.CDLL(LIB)
    L.m3_get_limits.restype = Limits
    L.m3_get_limits.argtypes = []
    L.m3_status_string.restype = ctypes.c_char_p
    L.m3_status_string.argtypes = [ctypes.c_int]
    L.m3_workspace_bytes.restype = ctypes.c_size_t
    L.m3_workspace_bytes.argtypes = [ctypes.c_int, Dims, ctypes.c_int]
    L.m3_launch_count.restype = ctypes.c_uint64
    L.m3_launch_count.argtypes = []
    L.m3_device_error.restype = ctypes.c_int
    L.m3_device_error.argtypes = [_VP, ctypes.POINTER(ctypes.c_int)]
    L.m3_discretize.restype = ctypes.c_int
    L.m3_discretize.argtypes = [_VP, _VP, _VP, Dims, _VP, _VP, _VP, _VP]
    L.m3_rope_bc.restype = ctypes.c_int
    L.m3_rope_bc.argtypes = [_VP, _VP, ctypes.c_int, _VP, _VP, _VP, ctypes.POINTER(BcNorm), Dims,
                             _VP, _VP, _VP, _VP]
    L.m3_siso_chunked_fwd.restype = ctypes.c_int
    L.m3_siso_chunked_fwd.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                      ctypes.POINTER(BcNorm), _VP, _VP, _VP, Dims, _VP, _VP, _VP,
                                      _VP, _VP, ctypes.c_size_t, _VP]
    L.m3_mimo_chunked_fwd.restype = ctypes.c_int
    L.m3_mimo_chunked_fwd.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                      ctypes.c_int, ctypes.POINTER(BcNorm), _VP, _VP, _VP, Dims,
                                      _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP]
    L.m3_step_decode.restype = ctypes.c_int
    L.m3_step_decode.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                 ctypes.POINTER(BcNorm), Dims, _VP, _VP, _VP, _VP, _VP]
    for fn in (L.m3_mimo_step_decode, L.m3_step_decode_factored):
        fn.restype = ctypes.c_int
    L.m3_mimo_step_decode.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                      ctypes.POINTER(BcNorm), Dims, _VP, _VP, _VP, _VP, _VP]
    L.m3_step_decode_factored.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                          ctypes.POINTER(BcNorm), Dims, _VP, _VP, _VP, _VP, _VP, _VP]
    L.m3_selftest_bounded_wait.restype = ctypes.c_int
    L.m3_selftest_bounded_wait.argtypes = [_VP]
    L.m3_debug_fail_next_launches.restype = None
    L.m3_debug_fail_next_launches.argtypes = [ctypes.c_int]
    L.m3_chunked_bwd.restype = ctypes.c_int
    L.m3_chunked_bwd.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                 ctypes.POINTER(BcNorm), _VP, _VP, _VP, Dims, _VP, _VP, _VP, _VP,
                                 ctypes.POINTER(Grads), _VP, ctypes.c_size_t, _VP]
    _lib = L
    return L


def status_string(status):
    return lib().m3_status_string(int(status)).decode()


def launch_count():
    return int(lib().m3_launch_count())


def device_error(stream=None, with_site=False):
    """Synchronise the stream and return the device-side error status
    (M3_OK, or M3_ERR_TIMEOUT when a bounded wait inside a kernel gave up);
    with_site=True also returns the recorded wait site."""
    site = ctypes.c_int(0)
    st = int(lib().m3_device_error(_stream(stream), ctypes.byref(site)))
    return (st, site.value) if with_site else st


def selftest_bounded_wait(stream=None):
    """Enqueue the timeout-path self-test (one bounded wait that runs out after
    about a second); read the outcome with device_error()."""
    _check(lib().m3_selftest_bounded_wait(_stream(stream)), "m3_selftest_bounded_wait")


def debug_fail_next_launches(n):
    """Failure injection for tests: the next n library calls that pass their
    argument checks fail with M3_ERR_CUDA (raised as M3Error here) and
    launch nothing.  n <= 0 turns it off."""
    lib().m3_debug_fail_next_launches(int(n))


def limits():
    l = lib().m3_get_limits()
    return dict(max_dstate=l.max_dstate, max_headdim=l.max_headdim,
                max_state_elems=l.max_state_elems, max_rank=l.max_rank)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _expect(where, dev, name, t, numel, dtype, required=True):
    """The library sees only pointers and the sizes in m3_dims, so the binding
    checks each tensor against those sizes (element count, dtype, device)
    before the call: a tensor shorter than the sizes say would otherwise be
    read or written past its end."""
    if t is None:
        if required:
            raise ValueError("%s: %s is required" % (where, name))
        return
    if t.numel() != numel:
        raise ValueError("%s: %s has %d elements (shape %s), the sizes need %d"
                         % (where, name, t.numel(), tuple(t.shape), numel))
    if t.dtype != dtype:
        raise ValueError("%s: %s is %s, expected %s" % (where, name, t.dtype, dtype))
    if t.device != dev:
        raise ValueError("%s: %s is on %s, expected %s" % (where, name, t.device, dev))


def _io_dtype(where, t):
    if t.dtype not in _DTYPE:
        raise ValueError("%s: x, B, C must be float32 or bfloat16, got %s" % (where, t.dtype))
    return t.dtype


def _expect_norm(where, dev, norm, H, R, N):
    if norm is None:
        return
    for k in ("normw_B", "normw_C"):
        _expect(where, dev, k, norm.get(k), N, torch.float32, required=False)
    for k in ("bias_B", "bias_C"):
        _expect(where, dev, k, norm.get(k), H * R * N, torch.float32, required=False)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _norm(norm):
    if norm is None:
        return None, ()
    keep = tuple(norm.get(k) for k in ("normw_B", "normw_C", "bias_B", "bias_C"))
    s = BcNorm(*[_ptr(k) for k in keep], float(norm.get("eps", 1e-5)))
    return ctypes.byref(s), keep + (s,)


def _check(rc, where):
    if rc != M3_OK:
        raise M3Error(rc, where)


def workspace_bytes(which, dims, dtype):
    return int(lib().m3_workspace_bytes(int(which), dims, int(dtype)))


def discretize(dt, A, lam, out=None, stream=None):
    """S1: alpha, beta, gamma (Bt,T,H) fp32."""
    Bt, T, H = dt.shape
    al, be, ga = out if out is not None else tuple(torch.empty_like(dt) for _ in range(3))
    w, f, n, dev = "m3_discretize", torch.float32, Bt * T * H, dt.device
    for name, t in (("dt", dt), ("lam", lam), ("alpha", al), ("beta", be), ("gamma", ga)):
        _expect(w, dev, name, t, n, f)
    _expect(w, dev, "A", A, H, f)
    d = Dims(Bt, T, H, 1, 2, 1, 1, 0, 0)
    _check(lib().m3_discretize(_ptr(dt), _ptr(A), _ptr(lam), d, _ptr(al), _ptr(be), _ptr(ga),
                               _stream(stream)), "m3_discretize")
    return al, be, ga


def rope_bc(B, C, theta, dt, angle0=None, norm=None, out=None, stream=None):
    """S2: B_rot, C_rot (Bt,T,H,[R,]N), one row per head, dtype of B, and
    angle_final (Bt,H,K) fp32.  B, C are (Bt,T,G,N) or (Bt,T,G,R,N) with G
    dividing H; theta (Bt,T,H,K) gives H and the number K of rotated pairs."""
    if B.dim() == 4:
        Bt, T, G, N = B.shape
        R = 1
    else:
        Bt, T, G, R, N = B.shape
    H, K = theta.shape[2], theta.shape[3]
    if out is None:
        shape = (Bt, T, H, N) if B.dim() == 4 else (Bt, T, H, R, N)
        out = (torch.empty(shape, device=B.device, dtype=B.dtype),
               torch.empty(shape, device=B.device, dtype=B.dtype),
               torch.empty(Bt, H, K, device=B.device, dtype=torch.float32))
    Br, Cr, ang = out
    w, f, dev, io = "m3_rope_bc", torch.float32, B.device, _io_dtype("m3_rope_bc", B)
    _expect(w, dev, "C", C, B.numel(), io)
    _expect(w, dev, "theta", theta, Bt * T * H * K, f)
    _expect(w, dev, "dt", dt, Bt * T * H, f)
    _expect(w, dev, "angle0", angle0, Bt * H * K, f, required=False)
    _expect(w, dev, "B_rot", Br, Bt * T * H * R * N, io)
    _expect(w, dev, "C_rot", Cr, Bt * T * H * R * N, io)
    _expect(w, dev, "angle_final", ang, Bt * H * K, f, required=False)
    _expect_norm(w, dev, norm, H, R, N)
    nptr, keep = _norm(norm)
    d = Dims(Bt, T, H, 1, N, R, 1, G, K)
    _check(lib().m3_rope_bc(_ptr(B), _ptr(C), _DTYPE[B.dtype], _ptr(theta), _ptr(dt), _ptr(angle0),
                            nptr, d, _ptr(Br), _ptr(Cr), _ptr(ang), _stream(stream)), "m3_rope_bc")
    return Br, Cr, ang


def _state_outs(x, N, P, K, out):
    Bt, T, H = x.shape[0], x.shape[1], x.shape[2]
    if out is not None:
        return out
    dev = x.device
    return (torch.empty_like(x), torch.empty(Bt, H, N, P, device=dev, dtype=torch.float32),
            torch.empty(Bt, H, N, P, device=dev, dtype=torch.float32),
            torch.empty(Bt, H, K, device=dev, dtype=torch.float32))


def _expect_scan(w, x, dt, A, lam, theta, B, C, D, R, W_x=None, W_y=None, norm=None, h0=None, prevBx0=None,
                 angle0=None):
    """Element counts of the chunked scan's inputs: x (Bt,T,H,P); dt, lam
    (Bt,T,H); A, D (H); theta (Bt,T,H,K); B, C (Bt,T,G,[R,]N); W_x, W_y
    (H,R,P); h0, prevBx0 (Bt,H,N,P); angle0 (Bt,H,K)."""
    Bt, T, H, P = x.shape
    N, G, K = B.shape[-1], B.shape[2], theta.shape[-1]
    f, dev, io = torch.float32, x.device, _io_dtype(w, x)
    for name, t in (("dt", dt), ("lam", lam)):
        _expect(w, dev, name, t, Bt * T * H, f)
    for name, t in (("A", A), ("D", D)):
        _expect(w, dev, name, t, H, f)
    _expect(w, dev, "theta", theta, Bt * T * H * K, f)
    _expect(w, dev, "B", B, Bt * T * G * R * N, io)
    _expect(w, dev, "C", C, Bt * T * G * R * N, io)
    for name, t in (("W_x", W_x), ("W_y", W_y)):
        _expect(w, dev, name, t, H * R * P, f, required=False)
    for name, t in (("h0", h0), ("prevBx0", prevBx0)):
        _expect(w, dev, name, t, Bt * H * N * P, f, required=False)
    _expect(w, dev, "angle0", angle0, Bt * H * K, f, required=False)
    _expect_norm(w, dev, norm, H, R, N)
    return io


def _expect_state_outs(w, x, N, K, outs):
    Bt, T, H, P = x.shape
    y, hf, uf, af = outs
    f, dev = torch.float32, x.device
    _expect(w, dev, "y", y, x.numel(), x.dtype)
    _expect(w, dev, "h_final", hf, Bt * H * N * P, f, required=False)
    _expect(w, dev, "prevBx_final", uf, Bt * H * N * P, f, required=False)
    _expect(w, dev, "angle_final", af, Bt * H * K, f, required=False)


def _workspace(which, d, dtype, workspace, dev):
    need = workspace_bytes(which, d, dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None and workspace.device != dev:
        raise ValueError("workspace is on %s, expected %s" % (workspace.device, dev))
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return workspace, nbytes


def siso_chunked_fwd(x, dt, A, lam, theta, B, C, D, chunk, norm=None, h0=None, prevBx0=None,
                     angle0=None, workspace=None, out=None, stream=None):
    """S1+S2+S3: returns y (Bt,T,H,P), h_final, prevBx_final (Bt,H,N,P), angle_final
    (Bt,H,K).  B, C (Bt,T,G,N) with G dividing H; theta (Bt,T,H,K)."""
    Bt, T, H, P = x.shape
    N, G, K = B.shape[-1], B.shape[2], theta.shape[-1]
    w = "m3_siso_chunked_fwd"
    _expect_scan(w, x, dt, A, lam, theta, B, C, D, 1, norm=norm, h0=h0, prevBx0=prevBx0, angle0=angle0)
    y, hf, uf, af = _state_outs(x, N, P, K, out)
    _expect_state_outs(w, x, N, K, (y, hf, uf, af))
    d = Dims(Bt, T, H, P, N, 1, int(chunk), G, K)
    dtype = _DTYPE[x.dtype]
    ws, nbytes = _workspace(M3_WS_SISO, d, dtype, workspace, x.device)
    nptr, keep = _norm(norm)
    _check(lib().m3_siso_chunked_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(B),
                                     _ptr(C), _ptr(D), dtype, nptr, _ptr(h0), _ptr(prevBx0),
                                     _ptr(angle0), d, _ptr(y), _ptr(hf), _ptr(uf), _ptr(af),
                                     _ptr(ws), nbytes, _stream(stream)), "m3_siso_chunked_fwd")
    return y, hf, uf, af


def mimo_chunked_fwd(x, dt, A, lam, theta, B, C, D, chunk, W_x=None, W_y=None, norm=None, h0=None,
                     prevBx0=None, angle0=None, workspace=None, out=None, stream=None):
    """S4: B, C (Bt,T,G,R,N); W_x, W_y (H,R,P) or None for ones."""
    Bt, T, H, P = x.shape
    R, N, G, K = B.shape[-2], B.shape[-1], B.shape[2], theta.shape[-1]
    w = "m3_mimo_chunked_fwd"
    _expect_scan(w, x, dt, A, lam, theta, B, C, D, R, W_x, W_y, norm, h0, prevBx0, angle0)
    y, hf, uf, af = _state_outs(x, N, P, K, out)
    _expect_state_outs(w, x, N, K, (y, hf, uf, af))
    d = Dims(Bt, T, H, P, N, R, int(chunk), G, K)
    dtype = _DTYPE[x.dtype]
    ws, nbytes = _workspace(M3_WS_MIMO, d, dtype, workspace, x.device)
    nptr, keep = _norm(norm)
    _check(lib().m3_mimo_chunked_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(B),
                                     _ptr(C), _ptr(D), _ptr(W_x), _ptr(W_y), dtype, nptr, _ptr(h0),
                                     _ptr(prevBx0), _ptr(angle0), d, _ptr(y), _ptr(hf), _ptr(uf),
                                     _ptr(af), _ptr(ws), nbytes, _stream(stream)),
           "m3_mimo_chunked_fwd")
    return y, hf, uf, af


def _expect_decode(w, x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, R, y, h, angle, W_x=None, W_y=None,
                   norm=None):
    """Element counts of a decode step's arguments: x_t, y (Bt,H,P); dt_t,
    lam_t (Bt,H); A, D (H); theta_t, angle (Bt,H,K); B_t, C_t (Bt,G,[R,]N);
    W_x, W_y (H,R,P); h (Bt,H,N,P)."""
    Bt, H, P = x_t.shape
    N, G, K = B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    f, dev, io = torch.float32, x_t.device, _io_dtype(w, x_t)
    for name, t in (("dt_t", dt_t), ("lam_t", lam_t)):
        _expect(w, dev, name, t, Bt * H, f)
    for name, t in (("A", A), ("D", D)):
        _expect(w, dev, name, t, H, f)
    _expect(w, dev, "theta_t", theta_t, Bt * H * K, f)
    _expect(w, dev, "B_t", B_t, Bt * G * R * N, io)
    _expect(w, dev, "C_t", C_t, Bt * G * R * N, io)
    for name, t in (("W_x", W_x), ("W_y", W_y)):
        _expect(w, dev, name, t, H * R * P, f, required=False)
    _expect(w, dev, "y_t", y, Bt * H * P, io)
    _expect(w, dev, "h", h, Bt * H * N * P, f)
    _expect(w, dev, "angle", angle, Bt * H * K, f)
    _expect_norm(w, dev, norm, H, R, N)


def step_decode(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, h, prevBx, angle, norm=None, y_out=None,
                stream=None):
    """S5: one decode step; B_t, C_t (Bt,G,N); theta_t (Bt,H,K); h, prevBx, angle
    are updated in place; returns y_t (Bt,H,P)."""
    Bt, H, P = x_t.shape
    N, G, K = B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    y = torch.empty_like(x_t) if y_out is None else y_out
    w = "m3_step_decode"
    _expect_decode(w, x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, 1, y, h, angle, norm=norm)
    _expect(w, x_t.device, "prevBx", prevBx, h.numel(), torch.float32)
    d = Dims(Bt, 1, H, P, N, 1, 1, G, K)
    nptr, keep = _norm(norm)
    _check(lib().m3_step_decode(_ptr(x_t), _ptr(dt_t), _ptr(A), _ptr(lam_t), _ptr(theta_t),
                                _ptr(B_t), _ptr(C_t), _ptr(D), _DTYPE[x_t.dtype], nptr, d, _ptr(h),
                                _ptr(prevBx), _ptr(angle), _ptr(y), _stream(stream)),
           "m3_step_decode")
    return y


def mimo_step_decode(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, h, prevBx, angle, W_x=None, W_y=None,
                     norm=None, y_out=None, stream=None):
    """S5 for rank R: one decode step on the full previous-input state.  B_t, C_t
    (Bt,G,R,N); h, prevBx, angle updated in place; returns y_t (Bt,H,P)."""
    Bt, H, P = x_t.shape
    R, N, G, K = B_t.shape[-2], B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    y = torch.empty_like(x_t) if y_out is None else y_out
    w = "m3_mimo_step_decode"
    _expect_decode(w, x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, R, y, h, angle, W_x, W_y, norm)
    _expect(w, x_t.device, "prevBx", prevBx, h.numel(), torch.float32)
    d = Dims(Bt, 1, H, P, N, R, 1, G, K)
    nptr, keep = _norm(norm)
    _check(lib().m3_mimo_step_decode(_ptr(x_t), _ptr(dt_t), _ptr(A), _ptr(lam_t), _ptr(theta_t), _ptr(B_t),
                                     _ptr(C_t), _ptr(D), _ptr(W_x), _ptr(W_y), _DTYPE[x_t.dtype], nptr, d,
                                     _ptr(h), _ptr(prevBx), _ptr(angle), _ptr(y), _stream(stream)),
           "m3_mimo_step_decode")
    return y


def step_decode_factored(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, h, b_prev, x_prev, angle, W_x=None,
                         W_y=None, norm=None, y_out=None, stream=None):
    """One decode step on the factored previous-input state (any rank; B_t, C_t
    (Bt,G,R,N)).  h, b_prev (Bt,H,R,N), x_prev (Bt,H,P) and angle are updated in
    place; returns y_t (Bt,H,P)."""
    Bt, H, P = x_t.shape
    R, N, G, K = B_t.shape[-2], B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    y = torch.empty_like(x_t) if y_out is None else y_out
    w = "m3_step_decode_factored"
    _expect_decode(w, x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, R, y, h, angle, W_x, W_y, norm)
    _expect(w, x_t.device, "b_prev", b_prev, Bt * H * R * N, torch.float32)
    _expect(w, x_t.device, "x_prev", x_prev, Bt * H * P, torch.float32)
    d = Dims(Bt, 1, H, P, N, R, 1, G, K)
    nptr, keep = _norm(norm)
    _check(lib().m3_step_decode_factored(_ptr(x_t), _ptr(dt_t), _ptr(A), _ptr(lam_t), _ptr(theta_t),
                                         _ptr(B_t), _ptr(C_t), _ptr(D), _ptr(W_x), _ptr(W_y),
                                         _DTYPE[x_t.dtype], nptr, d, _ptr(h), _ptr(b_prev), _ptr(x_prev),
                                         _ptr(angle), _ptr(y), _stream(stream)),
           "m3_step_decode_factored")
    return y


def chunked_bwd(x, dt, A, lam, theta, B, C, D, dy, chunk, W_x=None, W_y=None, norm=None, h0=None,
                prevBx0=None, angle0=None, dh_final=None, dprevBx_final=None, dangle_final=None,
                want=None, out=None, workspace=None, stream=None):
    """Backward of the chunked forward: returns a dict of fp32 gradients (the
    names in ``want``, by default all of them, without dW_x and dW_y for SISO;
    the gain and bias entries only when that part of the norm is on).  B, C
    (Bt,T,G,N) for SISO or (Bt,T,G,R,N) for rank R; dy has x's shape and dtype;
    the state adjoints default to zero.  ``out`` may hold preallocated fp32
    tensors by name (they are written and returned)."""
    Bt, T, H, P = x.shape
    R = B.shape[3] if B.dim() == 5 else 1
    N, G, K = B.shape[-1], B.shape[2], theta.shape[-1]
    mimo = B.dim() == 5
    w, f = "m3_chunked_bwd", torch.float32
    io = _expect_scan(w, x, dt, A, lam, theta, B, C, D, R, W_x, W_y, norm, h0, prevBx0, angle0)
    _expect(w, x.device, "dy", dy, x.numel(), io)
    for name, t, n in (("dh_final", dh_final, Bt * H * N * P), ("dprevBx_final", dprevBx_final, Bt * H * N * P),
                       ("dangle_final", dangle_final, Bt * H * K)):
        _expect(w, x.device, name, t, n, f, required=False)
    if want is None:
        want = tuple(k for k in GRAD_FIELDS if mimo or k not in ("dW_x", "dW_y"))
    dev = x.device
    shapes = dict(dx=x.shape, ddt=dt.shape, dA=A.shape, dlam=lam.shape, dtheta=theta.shape, dB=B.shape,
                  dC=C.shape, dD=D.shape, dW_x=(H, R, P), dW_y=(H, R, P), dnormw_B=(N,), dnormw_C=(N,),
                  dbias_B=(H, R, N), dbias_C=(H, R, N), dh0=(Bt, H, N, P), dprevBx0=(Bt, H, N, P),
                  dangle0=(Bt, H, K))
    nm = norm or {}
    off = {"dnormw_B": "normw_B", "dnormw_C": "normw_C", "dbias_B": "bias_B", "dbias_C": "bias_C"}
    pre = out or {}
    out = {k: (pre[k] if k in pre else torch.empty(shapes[k], device=dev, dtype=torch.float32)) for k in want
           if k not in off or nm.get(off[k]) is not None}
    for k, t in out.items():
        n = 1
        for e in shapes[k]:
            n *= e
        _expect(w, dev, k, t, n, f)
    g = Grads(*[_ptr(out.get(k)) for k in GRAD_FIELDS])
    d = Dims(Bt, T, H, P, N, R if mimo else 1, int(chunk), G, K)
    dtype = _DTYPE[x.dtype]
    ws, nbytes = _workspace(M3_WS_BWD_MIMO if mimo else M3_WS_BWD_SISO, d, dtype, workspace, dev)
    nptr, keep = _norm(norm)
    _check(lib().m3_chunked_bwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(W_x), _ptr(W_y), dtype, nptr, _ptr(h0), _ptr(prevBx0), _ptr(angle0), d,
                                _ptr(dy), _ptr(dh_final), _ptr(dprevBx_final), _ptr(dangle_final),
                                ctypes.byref(g), _ptr(ws), nbytes, _stream(stream)), "m3_chunked_bwd")
    return out
