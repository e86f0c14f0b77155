"""The seeded input generators (CPU): every draw is reproducible from its seed,
has the stated shape, dtype and range, and the grouped / partial-RoPE
options change only the shapes of B, C and theta, not the other draws."""
import math

import torch

from state_space_lm_b200 import inputs as gen


def test_same_seed_same_bytes_and_shapes():
    a = gen.scan_inputs(2, 33, 4, 8, 16, rank=3, dtype="bf16", seed=123, mimo_weights=True, bcnorm=True)
    b = gen.scan_inputs(2, 33, 4, 8, 16, rank=3, dtype="bf16", seed=123, mimo_weights=True, bcnorm=True)
    for k, v in a.items():
        if isinstance(v, torch.Tensor):
            assert torch.equal(v, b[k]), k
    assert a["x"].shape == (2, 33, 4, 8) and a["x"].dtype == torch.bfloat16
    assert a["B"].shape == (2, 33, 4, 3, 16) and a["B"].dtype == torch.bfloat16
    assert a["theta"].shape == (2, 33, 4, 8) and a["theta"].dtype == torch.float32
    assert a["Wx"].shape == (4, 3, 8) and a["bias_B"].shape == (4, 3, 16)


def test_value_ranges():
    a = gen.scan_inputs(4, 256, 8, 16, 32, dtype="f32", seed=7)
    assert bool((a["dt"] > 0).all())                                  # softplus
    assert bool(((a["lam"] > 0) & (a["lam"] < 1)).all())              # sigmoid
    assert bool((a["A"] < 0).all()) and bool((a["A"] >= -math.e).all())  # -exp(U(0,1))
    assert float(a["theta"].abs().max()) <= math.pi / 8
    assert abs(float(a["B"].std()) - 1 / math.sqrt(32)) < 0.02        # N(0,1)/sqrt(N)


def test_groups_and_pairs_change_only_their_shapes():
    full = gen.scan_inputs(2, 10, 4, 8, 16, dtype="f32", seed=9)
    grp = gen.scan_inputs(2, 10, 4, 8, 16, dtype="f32", seed=9, ngroups=2, rope_pairs=3)
    assert grp["B"].shape == (2, 10, 2, 16) and grp["theta"].shape == (2, 10, 4, 3)
    for k in ("x", "dt", "A", "lam"):
        assert torch.equal(full[k], grp[k]), k


def test_workload_configs_and_decode_steps():
    for idx, c in gen.CONFIGS.items():
        assert c["dstate"] % 2 == 0 and c["nheads"] % (c.get("ngroups") or c["nheads"]) == 0, idx
    g = gen.make_generator(1)
    st = gen.decode_step_inputs(g, 3, 4, 8, 16, rank=2, ngroups=2, rope_pairs=5)
    assert st["B"].shape == (3, 2, 2, 16) and st["theta"].shape == (3, 4, 5) and st["x"].shape == (3, 4, 8)
    dy = gen.grad_seed(torch.zeros(2, 3, 4, 5, dtype=torch.bfloat16), 11)
    assert dy.dtype == torch.bfloat16 and torch.equal(dy, gen.grad_seed(torch.zeros(2, 3, 4, 5,
                                                                                    dtype=torch.bfloat16), 11))
