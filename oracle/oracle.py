"""ctypes wrapper around the fp64 C oracle (``m3_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Arrays are float64 numpy arrays in the layouts
the C file documents (row-major, last index fastest):

    x, y (Bt,T,H,P); dt, lam (Bt,T,H); A, D (H); theta (Bt,T,H,N/2);
    B, C (Bt,T,H,N) for SISO or (Bt,T,H,R,N) for MIMO; W_x, W_y (H,R,P);
    h, prev_Bx (Bt,H,N,P); angle (Bt,H,N/2).

Inputs stored in bf16 or fp32 are widened to float64 by the caller before
they reach the oracle, so the oracle sees exactly the values the GPU sees.
"""
import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libm3_oracle.so")
_lib = None


def oracle_lib_path():
    return _LIB


def compile_source(src, out):
    """gcc, plain -O2: no fast-math and no FMA contraction."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
           "-pthread", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_oracle(force=False):
    """Compile the oracle (once; again when the source is newer)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    return compile_source(_SRC, _LIB)


def oracle_source_path():
    return _SRC


class _Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_long), ("seqlen", ctypes.c_long),
                ("nheads", ctypes.c_long), ("headdim", ctypes.c_long),
                ("dstate", ctypes.c_long), ("rank", ctypes.c_long),
                ("ngroups", ctypes.c_long), ("rope_pairs", ctypes.c_long)]


GRAD_NAMES = ("dx", "ddt", "dA", "dlam", "dtheta", "dB", "dC", "dD", "dWx", "dWy",
              "dnormw_B", "dnormw_C", "dbias_B", "dbias_C", "dh0", "dprevBx0", "dangle0")


class _Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_NAMES]


class _Norm(ctypes.Structure):
    _fields_ = [("normw_B", ctypes.c_void_p), ("normw_C", ctypes.c_void_p),
                ("bias_B", ctypes.c_void_p), ("bias_C", ctypes.c_void_p),
                ("eps", ctypes.c_double)]


def _open(path):
    lib = ctypes.CDLL(path)
    for name in ("m3o_discretize", "m3o_rope_bc", "m3o_siso_loop", "m3o_mimo_loop",
                 "m3o_siso_chunked", "m3o_step_decode", "m3o_mimo_step_decode", "m3o_step_decode_factored",
                 "m3o_mimo_loop_bwd"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _open(build_oracle())
    return _lib


@contextlib.contextmanager
def use_library(path):
    """Temporarily route every oracle call to another build of m3_oracle.c
    (the mutation test uses this to check that planted mistakes are caught)."""
    global _lib
    saved = _load()
    _lib = _open(path)
    try:
        yield
    finally:
        _lib = saved


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _norm(norm):
    """norm: None or dict(normw_B, normw_C, bias_B, bias_C, eps)."""
    if norm is None:
        return None, []
    keep = [_f64(norm.get(k)) for k in ("normw_B", "normw_C", "bias_B", "bias_C")]
    s = _Norm(*[_p(k) for k in keep], float(norm.get("eps", 1e-5)))
    return ctypes.byref(s), keep + [s]


def _dims(Bt, T, H, P, N, R=1, G=0, K=0):
    """G: B/C groups (0 or H: one per head); K: rotated pairs (0 or N/2: all)."""
    return _Dims(Bt, T, H, P, N, R, G, K)


def discretize(dt, A, lam):
    """alpha, beta, gamma, each (Bt,T,H)."""
    dt, A, lam = _f64(dt), _f64(A), _f64(lam)
    Bt, T, H = dt.shape
    al, be, ga = (np.empty_like(dt) for _ in range(3))
    L = ctypes.c_long   # long parameters: ctypes would pass a bare int as a C int
    rc = _load().m3o_discretize(_p(dt), _p(A), _p(lam), L(Bt), L(T), L(H), _p(al), _p(be), _p(ga))
    assert rc == 0
    return al, be, ga


def rope_bc(B, C, theta, dt, angle0=None, norm=None):
    """B_rot, C_rot per head (Bt,T,H,[R,]N), angle_final (Bt,H,K).

    B, C may be (Bt,T,G,N) or (Bt,T,G,R,N) with G dividing H; theta (Bt,T,H,K)
    gives H and the number K of rotated pairs."""
    B, C, theta, dt, angle0 = _f64(B), _f64(C), _f64(theta), _f64(dt), _f64(angle0)
    if B.ndim == 4:
        Bt, T, G, N = B.shape
        R = 1
    else:
        Bt, T, G, R, N = B.shape
    H, K = theta.shape[2], theta.shape[3]
    shape = (Bt, T, H, N) if B.ndim == 4 else (Bt, T, H, R, N)
    Br, Cr = np.empty(shape), np.empty(shape)
    ang = np.empty((Bt, H, K))
    nptr, keep = _norm(norm)
    rc = _load().m3o_rope_bc(_p(B), _p(C), _p(theta), _p(dt), _p(angle0), nptr,
                             _dims(Bt, T, H, 1, N, R, G, K), _p(Br), _p(Cr), _p(ang))
    assert rc == 0
    return Br, Cr, ang


def siso_loop(x, dt, A, lam, theta, B, C, D, h0=None, prevBx0=None, angle0=None,
              norm=None, nthreads=0, return_threads=False):
    """Sequential SISO scan. Returns y, h_final, prev_Bx, angle_final."""
    x, dt, A, lam, theta, B, C, D = (_f64(a) for a in (x, dt, A, lam, theta, B, C, D))
    h0, prevBx0, angle0 = _f64(h0), _f64(prevBx0), _f64(angle0)
    Bt, T, H, P = x.shape
    N, G, K = B.shape[-1], B.shape[2], theta.shape[-1]
    y = np.empty_like(x)
    hf = np.empty((Bt, H, N, P))
    uf = np.empty((Bt, H, N, P))
    af = np.empty((Bt, H, K))
    nptr, keep = _norm(norm)
    rc = _load().m3o_siso_loop(_p(x), _p(dt), _p(A), _p(lam), _p(theta), _p(B), _p(C), _p(D),
                               nptr, _p(h0), _p(prevBx0), _p(angle0), _dims(Bt, T, H, P, N, 1, G, K),
                               _p(y), _p(hf), _p(uf), _p(af), int(nthreads))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    out = (y, hf, uf, af)
    return (out, rc) if return_threads else out


def mimo_loop(x, dt, A, lam, theta, B, C, D, Wx=None, Wy=None, h0=None, prevBx0=None,
              angle0=None, norm=None, nthreads=0, return_threads=False):
    """Sequential rank-R MIMO scan. B, C (Bt,T,G,R,N). Returns y, h, prev_Bx, angle."""
    x, dt, A, lam, theta, B, C, D = (_f64(a) for a in (x, dt, A, lam, theta, B, C, D))
    Wx, Wy, h0, prevBx0, angle0 = (_f64(a) for a in (Wx, Wy, h0, prevBx0, angle0))
    Bt, T, H, P = x.shape
    R, N, G, K = B.shape[-2], B.shape[-1], B.shape[2], theta.shape[-1]
    y = np.empty_like(x)
    hf = np.empty((Bt, H, N, P))
    uf = np.empty((Bt, H, N, P))
    af = np.empty((Bt, H, K))
    nptr, keep = _norm(norm)
    rc = _load().m3o_mimo_loop(_p(x), _p(dt), _p(A), _p(lam), _p(theta), _p(B), _p(C), _p(D),
                               _p(Wx), _p(Wy), nptr, _p(h0), _p(prevBx0), _p(angle0),
                               _dims(Bt, T, H, P, N, R, G, K), _p(y), _p(hf), _p(uf), _p(af),
                               int(nthreads))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    out = (y, hf, uf, af)
    return (out, rc) if return_threads else out


def siso_chunked(x, dt, A, lam, theta, B, C, D, chunk, h0=None, prevBx0=None, angle0=None,
                 norm=None, nthreads=0):
    """fp64 chunked form (self-test of the shifted-gamma fold)."""
    x, dt, A, lam, theta, B, C, D = (_f64(a) for a in (x, dt, A, lam, theta, B, C, D))
    h0, prevBx0, angle0 = _f64(h0), _f64(prevBx0), _f64(angle0)
    Bt, T, H, P = x.shape
    N, G, K = B.shape[-1], B.shape[2], theta.shape[-1]
    y = np.empty_like(x)
    hf = np.empty((Bt, H, N, P))
    uf = np.empty((Bt, H, N, P))
    af = np.empty((Bt, H, K))
    nptr, keep = _norm(norm)
    rc = _load().m3o_siso_chunked(_p(x), _p(dt), _p(A), _p(lam), _p(theta), _p(B), _p(C),
                                  _p(D), nptr, _p(h0), _p(prevBx0), _p(angle0),
                                  _dims(Bt, T, H, P, N, 1, G, K), ctypes.c_long(int(chunk)), _p(y), _p(hf), _p(uf),
                                  _p(af), int(nthreads))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    return y, hf, uf, af


def step_decode(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, h, prevBx, angle, norm=None,
                nthreads=0):
    """One SISO decode step. Per-token inputs: x_t (Bt,H,P), dt_t/lam_t (Bt,H),
    theta_t (Bt,H,K), B_t/C_t (Bt,G,N).  Returns y_t (Bt,H,P), h, prev_Bx, angle
    (new arrays; the inputs are not modified)."""
    x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D = (
        _f64(a) for a in (x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D))
    h, prevBx, angle = (np.array(a, dtype=np.float64, copy=True) for a in (h, prevBx, angle))
    Bt, H, P = x_t.shape
    N, G, K = B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    y = np.empty((Bt, 1, H, P))
    nptr, keep = _norm(norm)
    rc = _load().m3o_step_decode(_p(x_t), _p(dt_t), _p(A), _p(lam_t), _p(theta_t), _p(B_t),
                                 _p(C_t), _p(D), nptr, _dims(Bt, 1, H, P, N, 1, G, K), _p(h), _p(prevBx),
                                 _p(angle), _p(y), int(nthreads))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    return y[:, 0], h, prevBx, angle


def mimo_step_decode(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, h, prevBx, angle, Wx=None, Wy=None,
                     norm=None, nthreads=0):
    """One rank-R MIMO decode step on the full previous-input state.  B_t, C_t
    (Bt,G,R,N).  Returns y_t (Bt,H,P), h, prev_Bx, angle (new arrays)."""
    x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, Wx, Wy = (
        _f64(a) for a in (x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, Wx, Wy))
    h, prevBx, angle = (np.array(a, dtype=np.float64, copy=True) for a in (h, prevBx, angle))
    Bt, H, P = x_t.shape
    R, N, G, K = B_t.shape[-2], B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    y = np.empty((Bt, 1, H, P))
    nptr, keep = _norm(norm)
    rc = _load().m3o_mimo_step_decode(_p(x_t), _p(dt_t), _p(A), _p(lam_t), _p(theta_t), _p(B_t),
                                      _p(C_t), _p(D), _p(Wx), _p(Wy), nptr, _dims(Bt, 1, H, P, N, R, G, K),
                                      _p(h), _p(prevBx), _p(angle), _p(y), int(nthreads))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    return y[:, 0], h, prevBx, angle


def step_decode_factored(x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, h, bprev, xprev, angle,
                         Wx=None, Wy=None, norm=None):
    """One decode step on the factored previous-input state: bprev (Bt,H,R,N)
    is the rotated B of the previous token per rank and xprev (Bt,H,P) its x.
    B_t, C_t (Bt,G,R,N) (R = 1 for SISO); theta_t (Bt,H,K).  Returns y_t, h,
    bprev, xprev, angle (new arrays)."""
    x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, Wx, Wy = (
        _f64(a) for a in (x_t, dt_t, A, lam_t, theta_t, B_t, C_t, D, Wx, Wy))
    h, bprev, xprev, angle = (np.array(a, dtype=np.float64, copy=True) for a in (h, bprev, xprev, angle))
    Bt, H, P = x_t.shape
    R, N, G, K = B_t.shape[-2], B_t.shape[-1], B_t.shape[1], theta_t.shape[-1]
    y = np.empty((Bt, H, P))
    nptr, keep = _norm(norm)
    rc = _load().m3o_step_decode_factored(_p(x_t), _p(dt_t), _p(A), _p(lam_t), _p(theta_t), _p(B_t),
                                          _p(C_t), _p(D), _p(Wx), _p(Wy), nptr, _dims(Bt, 1, H, P, N, R, G, K),
                                          _p(h), _p(bprev), _p(xprev), _p(angle), _p(y))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    return y, h, bprev, xprev, angle


def loop_bwd(x, dt, A, lam, theta, B, C, D, dy=None, Wx=None, Wy=None, h0=None, prevBx0=None,
             angle0=None, norm=None, dh=None, dprevBx=None, dangle=None):
    """Gradients of L = <dy, y> + <dh, h_final> + <dprevBx, prevBx_final> +
    <dangle, angle_final> with respect to every input of the scan (SISO when B
    is (Bt,T,G,N), rank R when it is (Bt,T,G,R,N)).  Returns a dict keyed by
    GRAD_NAMES (dWx, dWy are the gradients for all-ones vectors when Wx, Wy
    are None; the norm entries are None when that part of the norm is off)."""
    x, dt, A, lam, theta, B, C, D = (_f64(a) for a in (x, dt, A, lam, theta, B, C, D))
    Wx, Wy, h0, prevBx0, angle0 = (_f64(a) for a in (Wx, Wy, h0, prevBx0, angle0))
    dy, dh, dprevBx, dangle = (_f64(a) for a in (dy, dh, dprevBx, dangle))
    Bt, T, H, P = x.shape
    R = B.shape[3] if B.ndim == 5 else 1
    N, G, K = B.shape[-1], B.shape[2], theta.shape[-1]
    shapes = dict(dx=x.shape, ddt=dt.shape, dA=(H,), dlam=lam.shape, dtheta=theta.shape, dB=B.shape,
                  dC=C.shape, dD=(H,), dWx=(H, R, P), dWy=(H, R, P), dnormw_B=(N,), dnormw_C=(N,),
                  dbias_B=(H, R, N), dbias_C=(H, R, N), dh0=(Bt, H, N, P), dprevBx0=(Bt, H, N, P),
                  dangle0=(Bt, H, K))
    out = {k: np.zeros(v) for k, v in shapes.items()}
    nm = norm or {}
    for k, key in (("dnormw_B", "normw_B"), ("dnormw_C", "normw_C"), ("dbias_B", "bias_B"),
                   ("dbias_C", "bias_C")):
        if nm.get(key) is None:
            out[k] = None
    g = _Grads(*[_p(out[k]) for k in GRAD_NAMES])
    nptr, keep = _norm(norm)
    rc = _load().m3o_mimo_loop_bwd(_p(x), _p(dt), _p(A), _p(lam), _p(theta), _p(B), _p(C), _p(D), _p(Wx),
                                   _p(Wy), nptr, _p(h0), _p(prevBx0), _p(angle0),
                                   _dims(Bt, T, H, P, N, R, G, K), _p(dy), _p(dh), _p(dprevBx), _p(dangle),
                                   ctypes.byref(g))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    return out
