"""Seeded synthetic inputs for the Mamba-3 scan.

This module only draws random numbers; it holds none of the scan's arithmetic.
Both the CUDA path and the fp64 oracle consume the tensors it returns (the
oracle after widening the stored values to float64), so the two see the same
bytes.

Recipe (the pages publish no dataset for this path; the shapes stand in for
the workloads they describe -- 16 heads, headdim 64, d_model 1024 from the
Mamba-3-Lite "Model reference" page, dState 128 and 32 heads from the
370M checkpoint in the dotLLM pull request):

    x ~ N(0,1)                 dt  = softplus(N(0,1) + dt_shift)
    A = -exp(U(0,1)) per head   lam = sigmoid(N(0,1))
    theta ~ U(-pi/8, pi/8)      B, C ~ N(0,1) / sqrt(N)
    D ~ N(0,1) per head         W_x, W_y = 1 + 0.02 N(0,1)   (MIMO)

Every value is drawn in float64 from one ``torch.Generator`` seeded once, in
the fixed order x, dt, A, lam, theta, B, C, D, W_x, W_y, then the optional
QkNorm/bias parameters, then the per-step decode inputs; it is rounded once to
its storage dtype (bf16 or fp32 for x, B, C; fp32 for everything else).
"""
import math

import torch

SEED_BASE = 20261202

# The five workloads.  "chunk" is the chunk length of the chunked algorithm.
CONFIGS = {
    0: dict(name="tiny_siso_fp32", batch=1, seqlen=64, nheads=2, headdim=4, dstate=4,
            rank=1, chunk=16, dtype="f32", dt_shift=-2.0),
    1: dict(name="siso_8x2048_h16_p64_n128", batch=8, seqlen=2048, nheads=16, headdim=64,
            dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0),
    2: dict(name="mimo_r4_8x2048_h16_p64_n128", batch=8, seqlen=2048, nheads=16, headdim=64,
            dstate=128, rank=4, chunk=64, dtype="bf16", dt_shift=-2.0),
    3: dict(name="siso_long_1x32768_h32_p64_n128", batch=1, seqlen=32768, nheads=32,
            headdim=64, dstate=128, rank=1, chunk=128, dtype="bf16", dt_shift=-4.0),
    4: dict(name="decode_512xh16_p64_n128", batch=512, seqlen=256, nheads=16, headdim=64,
            dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0, steps=1024),
    # decode on the factored previous-input state (b_prev, x_prev), SISO and rank 4
    5: dict(name="decode_factored_512xh16_p64_n128", batch=512, seqlen=256, nheads=16, headdim=64,
            dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0, steps=1024, state="factored"),
    6: dict(name="decode_factored_mimo_r4_512xh16_p64_n128", batch=512, seqlen=256, nheads=16,
            headdim=64, dstate=128, rank=4, chunk=64, dtype="bf16", dt_shift=-2.0, steps=1024,
            state="factored"),
    # one B/C group shared by all heads and 32 rotated pairs of 64 (the 370M
    # checkpoint's n_groups 1 and rope fraction 0.5), default workload's shape
    7: dict(name="siso_g1_rope32_8x2048_h16_p64_n128", batch=8, seqlen=2048, nheads=16, headdim=64,
            dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0, ngroups=1, rope_pairs=32),
    # the backward (all input gradients) of the default workload
    8: dict(name="bwd_siso_8x2048_h16_p64_n128", batch=8, seqlen=2048, nheads=16, headdim=64,
            dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0, grad=True),
    # the standalone prep passes: S1 alone (alpha, beta, gamma out) over the
    # decode workload's 512 sequences at the default 2048 tokens (the default
    # batch's dt and lam, 2 MB, would sit in L2), and S2 alone (rotated B, C and
    # the angle out) on the default workload's inputs
    9: dict(name="discretize_512x2048_h16", batch=512, seqlen=2048, nheads=16, headdim=64,
            dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0, prep="discretize"),
    10: dict(name="rope_bc_8x2048_h16_n128", batch=8, seqlen=2048, nheads=16, headdim=64,
             dstate=128, rank=1, chunk=64, dtype="bf16", dt_shift=-2.0, prep="rope"),
}

_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def storage_dtype(name):
    return _DTYPES[name]


def make_generator(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal(g, shape):
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _uniform(g, shape, lo, hi):
    return torch.rand(*shape, generator=g, dtype=torch.float64) * (hi - lo) + lo


def scan_inputs(batch, seqlen, nheads, headdim, dstate, rank=1, dtype="bf16",
                dt_shift=-2.0, seed=SEED_BASE, mimo_weights=None, bcnorm=False,
                generator=None, ngroups=0, rope_pairs=0):
    """Inputs of one chunked-scan call, as CPU tensors in their storage dtype.

    Returns a dict with x (Bt,T,H,P), dt (Bt,T,H), A (H), lam (Bt,T,H),
    theta (Bt,T,H,K), B and C ((Bt,T,G,N) when rank == 1 and mimo_weights is
    falsy, else (Bt,T,G,R,N)), D (H), and, for MIMO, Wx and Wy (H,R,P).
    G = ngroups and K = rope_pairs, 0 meaning H and N/2 (the draws are the
    same in number and order; only these shapes change).
    With bcnorm=True it adds normw_B, normw_C (N), bias_B, bias_C (H,R,N) and
    eps.  The generator is returned under "generator" so that later draws
    (decode steps) continue the same stream.
    """
    g = generator if generator is not None else make_generator(seed)
    sdt = _DTYPES[dtype]
    Bt, T, H, P, N, R = batch, seqlen, nheads, headdim, dstate, rank
    G, K = ngroups or H, rope_pairs or N // 2
    mimo = bool(mimo_weights) if mimo_weights is not None else R > 1
    bc_shape = (Bt, T, G, R, N) if mimo else (Bt, T, G, N)
    out = {}
    out["x"] = _normal(g, (Bt, T, H, P)).to(sdt)
    out["dt"] = torch.nn.functional.softplus(_normal(g, (Bt, T, H)) + dt_shift).float()
    out["A"] = (-torch.exp(_uniform(g, (H,), 0.0, 1.0))).float()
    out["lam"] = torch.sigmoid(_normal(g, (Bt, T, H))).float()
    out["theta"] = _uniform(g, (Bt, T, H, K), -math.pi / 8, math.pi / 8).float()
    out["B"] = (_normal(g, bc_shape) / math.sqrt(N)).to(sdt)
    out["C"] = (_normal(g, bc_shape) / math.sqrt(N)).to(sdt)
    out["D"] = _normal(g, (H,)).float()
    if mimo:
        out["Wx"] = (1.0 + 0.02 * _normal(g, (H, R, P))).float()
        out["Wy"] = (1.0 + 0.02 * _normal(g, (H, R, P))).float()
    if bcnorm:
        out["normw_B"] = (1.0 + 0.1 * _normal(g, (N,))).float()
        out["normw_C"] = (1.0 + 0.1 * _normal(g, (N,))).float()
        out["bias_B"] = (0.1 * _normal(g, (H, R, N))).float()
        out["bias_C"] = (0.1 * _normal(g, (H, R, N))).float()
        out["eps"] = 1e-5
    out["generator"] = g
    return out


def decode_step_inputs(generator, batch, nheads, headdim, dstate, dtype="bf16",
                       dt_shift=-2.0, rank=1, rank_axis=False, ngroups=0, rope_pairs=0):
    """Per-token inputs of one decode step, drawn from ``generator``:
    x_t (Bt,H,P), dt_t (Bt,H), lam_t (Bt,H), theta_t (Bt,H,K), B_t and C_t
    (Bt,G,N), or (Bt,G,R,N) when rank > 1 or rank_axis (G = ngroups or H,
    K = rope_pairs or N/2)."""
    g = generator
    sdt = _DTYPES[dtype]
    Bt, H, P, N = batch, nheads, headdim, dstate
    G, K = ngroups or H, rope_pairs or N // 2
    bc = (Bt, G, rank, N) if (rank > 1 or rank_axis) else (Bt, G, N)
    out = {}
    out["x"] = _normal(g, (Bt, H, P)).to(sdt)
    out["dt"] = torch.nn.functional.softplus(_normal(g, (Bt, H)) + dt_shift).float()
    out["lam"] = torch.sigmoid(_normal(g, (Bt, H))).float()
    out["theta"] = _uniform(g, (Bt, H, K), -math.pi / 8, math.pi / 8).float()
    out["B"] = (_normal(g, bc) / math.sqrt(N)).to(sdt)
    out["C"] = (_normal(g, bc) / math.sqrt(N)).to(sdt)
    return out


def discretize_inputs(batch, seqlen, nheads, dt_shift=-2.0, seed=SEED_BASE):
    """Inputs of a standalone discretization: dt, lam (Bt,T,H) and A (H), drawn
    from one generator in the order dt, A, lam with the laws above."""
    g = make_generator(seed)
    Bt, T, H = batch, seqlen, nheads
    out = {}
    out["dt"] = torch.nn.functional.softplus(_normal(g, (Bt, T, H)) + dt_shift).float()
    out["A"] = (-torch.exp(_uniform(g, (H,), 0.0, 1.0))).float()
    out["lam"] = torch.sigmoid(_normal(g, (Bt, T, H))).float()
    out["generator"] = g
    return out


def config_inputs(idx, seed=None, **overrides):
    """Inputs of workload ``idx`` (0-3, 7 and 8: one chunked-scan call, forward
    or backward; 4-6: the prefill of a decode workload -- its steps come from
    ``decode_step_inputs`` with the returned generator; 9: dt, A, lam of a
    standalone discretization; 10: a chunked-scan call's inputs, of which the
    standalone rotation uses B, C, theta and dt).  The backward's dy is drawn
    by ``grad_seed``."""
    c = dict(CONFIGS[idx])
    c.update(overrides)
    s = SEED_BASE + idx if seed is None else seed
    if c.get("prep") == "discretize":
        return discretize_inputs(c["batch"], c["seqlen"], c["nheads"], dt_shift=c["dt_shift"], seed=s)
    return scan_inputs(c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"],
                       rank=c["rank"], dtype=c["dtype"], dt_shift=c["dt_shift"], seed=s,
                       mimo_weights=c["rank"] > 1, ngroups=c.get("ngroups", 0),
                       rope_pairs=c.get("rope_pairs", 0))


def grad_seed(x, seed):
    """dy ~ N(0, 1) in x's shape and dtype (the backward's output adjoint)."""
    g = make_generator(seed)
    return _normal(g, tuple(x.shape)).to(x.dtype)


def to_f64(t):
    """Widen a stored tensor to a float64 numpy array (what the oracle consumes)."""
    return t.detach().to("cpu", torch.float64).numpy()
