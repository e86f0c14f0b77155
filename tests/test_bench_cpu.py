"""bench.py's roofline arithmetic on CPU: the algorithmic bytes and flops of
each workload against the per-unit figures worked out by hand (inputs once,
outputs once, final states; causal-triangle flops)."""
import pytest

import bench
from state_space_lm_b200 import inputs as gen


def test_scan_bytes_default_workload():
    c = gen.CONFIGS[1]
    # 1032 B per token-head (x 128, B 256, C 256, theta 256, dt 4, lam 4, y 128)
    # + per lane h and prev_Bx (2 x 32 KB) and the angle (256 B) + A, D per head
    assert bench.scan_bytes(c) == 8 * 2048 * 16 * 1032 + 128 * (2 * 128 * 64 * 4 + 64 * 4) + 16 * 8
    assert bench.scan_bytes(c) == 278_954_112


def test_scan_bytes_mimo_and_grouped():
    c2 = gen.CONFIGS[2]
    per = 128 + 2 * 2 * 4 * 128 + 8 + 256 + 128          # 2568 B per token-head
    states = 128 * (2 * 128 * 64 * 4 + 64 * 4)
    params = 16 * 8 + 2 * 16 * 4 * 64 * 4
    assert bench.scan_bytes(c2) == 8 * 2048 * 16 * per + states + params
    c7 = gen.CONFIGS[7]                                   # one group, 32 rotated pairs
    per_head = 128 + 8 + 4 * 32 + 128
    per_group = 2 * 2 * 128
    states7 = 128 * (2 * 128 * 64 * 4 + 32 * 4)
    assert bench.scan_bytes(c7) == 8 * 2048 * (16 * per_head + 1 * per_group) + states7 + 16 * 8


def test_scan_flops_default_workload():
    # per 64-token chunk: 2 * pairs * (N + P) + 4 * Q * N * P + 2 * N * P, pairs = 64 * 65 / 2
    per_chunk = 2 * 2080 * (128 + 64) + 4 * 64 * 128 * 64 + 2 * 128 * 64
    assert bench.scan_flops(gen.CONFIGS[1]) == 128 * 32 * per_chunk
    assert bench.scan_flops(gen.CONFIGS[1]) == pytest.approx(11.93e9, rel=1e-3)


@pytest.mark.parametrize("idx,per_lane", [(4, 132_616), (5, 68_616), (6, 73_224)])
def test_decode_bytes(idx, per_lane):
    c = gen.CONFIGS[idx]
    extra = 2 * 16 * c["rank"] * 64 * 4 if c["rank"] > 1 else 0
    assert bench.decode_bytes(c) == 512 * 16 * per_lane + extra


def test_backward_bytes_and_flops():
    c = gen.CONFIGS[8]
    # reads: x, dy 256 + dt, lam 8 + theta 256 + B, C 512; writes: dx 256 + ddt, dlam 8 + dtheta 256
    # + dB, dC 1024 (fp32) = 2576 B per token-head
    states = 128 * (2 * 128 * 64 * 4 + 64 * 4)
    assert bench.bwd_bytes(c) == 8 * 2048 * 16 * 2576 + states + 16 * 16
    per_chunk = 12 * 64 * 128 * 64 + 2 * 2080 * (3 * 128 + 2 * 64)
    assert bench.bwd_flops(c) == 128 * 32 * per_chunk
    assert bench.bwd_flops(c) / (8 * 2048 * 16) == pytest.approx(131.6e3, rel=1e-3)
    assert bench.FFMA_PEAK_TFLOPS == pytest.approx(74.4, rel=1e-3)


def test_prep_bytes():
    # S1: dt, lam in, alpha, beta, gamma out (20 B per token-head) + A
    assert bench.prep_bytes(gen.CONFIGS[9]) == 512 * 2048 * 16 * 20 + 16 * 4
    # S2: B, C in (512), theta (256), dt (4), rotated B, C out (512) = 1284 B
    # per token-head, + the final angle per lane
    assert bench.prep_bytes(gen.CONFIGS[10]) == 8 * 2048 * 16 * 1284 + 128 * 64 * 4
