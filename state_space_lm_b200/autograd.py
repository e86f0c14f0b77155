"""Differentiable Mamba-3 scan for PyTorch: the chunked forward and
m3_chunked_bwd behind one torch.autograd.Function.

Argument marshalling only: the forward calls m3_siso_chunked_fwd or
m3_mimo_chunked_fwd, the backward calls m3_chunked_bwd, and every gradient
comes from the CUDA library (there is no other implementation behind these
names).  The initial states and the final states take part in autograd too,
so a sequence can be split into pieces whose states are chained.
"""
import torch

from . import m3

_SEQ = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
_GRAD_OF = {"x": "dx", "dt": "ddt", "A": "dA", "lam": "dlam", "theta": "dtheta", "B": "dB", "C": "dC",
            "D": "dD", "W_x": "dW_x", "W_y": "dW_y", "h0": "dh0", "prevBx0": "dprevBx0", "angle0": "dangle0"}


class Mamba3Scan(torch.autograd.Function):
    """Inputs in the order of the C ABI; returns (y, h_final, prevBx_final,
    angle_final).  B, C with a rank axis (Bt,T,G,R,N) select the MIMO scan."""

    @staticmethod
    def forward(ctx, x, dt, A, lam, theta, B, C, D, W_x, W_y, h0, prevBx0, angle0, chunk):
        mimo = B.dim() == 5
        if not mimo and (W_x is not None or W_y is not None):
            raise ValueError("W_x, W_y need B and C with a rank axis (Bt,T,G,R,N)")
        if mimo:
            out = m3.mimo_chunked_fwd(x, dt, A, lam, theta, B, C, D, chunk, W_x=W_x, W_y=W_y, h0=h0,
                                      prevBx0=prevBx0, angle0=angle0)
        else:
            out = m3.siso_chunked_fwd(x, dt, A, lam, theta, B, C, D, chunk, h0=h0, prevBx0=prevBx0,
                                      angle0=angle0)
        ctx.save_for_backward(x, dt, A, lam, theta, B, C, D, W_x, W_y, h0, prevBx0, angle0)
        ctx.chunk = chunk
        ctx.mimo = mimo
        return out

    @staticmethod
    def backward(ctx, dy, dh, du, da):
        x, dt, A, lam, theta, B, C, D, W_x, W_y, h0, prevBx0, angle0 = ctx.saved_tensors
        inputs = dict(x=x, dt=dt, A=A, lam=lam, theta=theta, B=B, C=C, D=D, W_x=W_x, W_y=W_y, h0=h0,
                      prevBx0=prevBx0, angle0=angle0)
        names = ("x", "dt", "A", "lam", "theta", "B", "C", "D", "W_x", "W_y", "h0", "prevBx0", "angle0")
        want = tuple(_GRAD_OF[n] for n, need in zip(names, ctx.needs_input_grad[:13])
                     if need and (ctx.mimo or n not in ("W_x", "W_y")))
        if dy is None:
            dy = torch.zeros_like(x)
        cont = lambda t: None if t is None else t.contiguous()
        g = m3.chunked_bwd(x, dt, A, lam, theta, B, C, D, cont(dy.to(x.dtype)), ctx.chunk, W_x=W_x, W_y=W_y,
                           h0=h0, prevBx0=prevBx0, angle0=angle0, dh_final=cont(dh), dprevBx_final=cont(du),
                           dangle_final=cont(da), want=want)
        grads = []
        for n, need in zip(names, ctx.needs_input_grad[:13]):
            v = g.get(_GRAD_OF[n]) if need else None
            grads.append(None if v is None else v.to(inputs[n].dtype))
        return tuple(grads) + (None,)


def mamba3_scan(x, dt, A, lam, theta, B, C, D, chunk=64, W_x=None, W_y=None, h0=None, prevBx0=None,
                angle0=None):
    """Differentiable scan: returns y, h_final, prevBx_final, angle_final.
    Shapes and dtypes as in include/m3.h (x, B, C bf16 or fp32; the rest fp32)."""
    return Mamba3Scan.apply(x, dt, A, lam, theta, B, C, D, W_x, W_y, h0, prevBx0, angle0, chunk)
