"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case copies the oracle's C source, plants one plausible mistake (a
dropped factor, a wrong sign, a wrong index, a swapped operand), compiles the
copy and runs the pins of ``test_oracle_pins`` against it; at least one pin
must fail.  This shows the pins constrain every step of the oracle.
"""
import os

import numpy as np
import pytest

import test_oracle_grad_pins as gpins
import test_oracle_pins as pins

MUTATIONS = [
    ("beta without alpha", "double be = (1.0 - lm) * dl * al;", "double be = (1.0 - lm) * dl;"),
    ("gamma with alpha", "double ga = lm * dl;", "double ga = lm * dl * al;"),
    ("rotation sign", "out[2 * i] = c * v0 - s * v1;", "out[2 * i] = c * v0 + s * v1;"),
    ("dropped D skip", "yt[p] = acc + J->D[h] * xt[p];", "yt[p] = acc;"),
    ("swapped U terms", "hs[n * P + p] = al * hs[n * P + p] + be * Up[n * P + p] + ga * u;",
     "hs[n * P + p] = al * hs[n * P + p] + be * u + ga * Up[n * P + p];"),
    ("angle without dt", "phi[i] += dl * J->theta[bth * K + i];",
     "phi[i] += J->theta[bth * K + i];"),
    ("y from C transposed to B", "for (long n = 0; n < N; n++) acc += Cb[n] * hs[n * P + p];",
     "for (long n = 0; n < N; n++) acc += Bb[n] * hs[n * P + p];"),
    ("alpha sign", "double al = exp(dl * J->A[h]);\n        double be = (1.0 - lm) * dl * al;\n        double ga = lm * dl;\n        for (long i = 0; i < K; i++) phi[i] += dl * J->theta[bth * K + i];\n        bc_prepare",
     "double al = exp(-dl * J->A[h]);\n        double be = (1.0 - lm) * dl * al;\n        double ga = lm * dl;\n        for (long i = 0; i < K; i++) phi[i] += dl * J->theta[bth * K + i];\n        bc_prepare"),
    ("MIMO contract without W_y", "acc += (J->Wy ? J->Wy[(h * R + r) * P + p] : 1.0) * yr;", "acc += yr;"),
    ("chunk lookahead dropped", "sg = (1.0 - J->lam[nx]) * J->dt[nx];", "sg = 0.0;"),
    ("factored decode: previous term from the current x", "up += bp[r * N + n] * Xp[r * P + p];",
     "up += bp[r * N + n] * Xr[r * P + p];"),
    ("factored decode: b_prev not advanced", "memcpy(bprev + lane * R * N, Bb, sizeof(double) * R * N);", ""),
    ("groups interleaved instead of contiguous", "* G + h / (d.nheads / G)) * R + r)", "* G + h % G) * R + r)"),
    ("partial RoPE zeroes the unrotated pairs", "for (long n = 2 * K; n < N; n++) out[n] = v[n];",
     "for (long n = 2 * K; n < N; n++) out[n] = 0.0;"),
    ("partial RoPE rotates the last pairs", "double v0 = v[2 * i], v1 = v[2 * i + 1];\n        out[2 * i] = c * v0 - s * v1;\n        out[2 * i + 1] = s * v0 + c * v1;\n    }\n    for (long n = 2 * K; n < N; n++) out[n] = v[n];",
     "long j = i + N / 2 - K;\n        double v0 = v[2 * j], v1 = v[2 * j + 1];\n        out[2 * j] = c * v0 - s * v1;\n        out[2 * j + 1] = s * v0 + c * v1;\n    }\n    for (long n = 0; n < N - 2 * K; n++) out[n] = v[n];"),
    ("backward: beta adjoint from U_t", "dbe += gh * um;", "dbe += gh * u;"),
    ("backward: state adjoint not decayed", "Gh[k] = al[t] * Gh[k];", "Gh[k] = Gh[k];"),
    ("backward: angle adjoint sign", "gp += -db[2 * i] * bb[2 * i + 1] + db[2 * i + 1] * bb[2 * i];",
     "gp += db[2 * i] * bb[2 * i + 1] - db[2 * i + 1] * bb[2 * i];"),
    ("backward: pair adjoint rotated forward", "dBp[2 * i] = c * db[2 * i] + s * db[2 * i + 1];",
     "dBp[2 * i] = c * db[2 * i] - s * db[2 * i + 1];"),
    ("backward: QkNorm adjoint without the RMS term",
     "dsrc[n] += inv * ddst[n] * w[n] - src[n] * inv * inv * inv * s / (double)N;",
     "dsrc[n] += inv * ddst[n] * w[n];"),
    ("backward: lookahead adjoint dropped", "GU[n * P + p] = ga[t] * gh + GUf[n * P + p];",
     "GU[n * P + p] = ga[t] * gh;"),
    ("backward: dtheta without dt", "g->dtheta[bth * K + i] += dl * Gphi[i];", "g->dtheta[bth * K + i] += Gphi[i];"),
    ("backward: dt misses the angle term", "if (g->ddt) g->ddt[bth] += theta[bth * K + i] * Gphi[i];", ""),
    ("backward: a group's B rows overwritten, not summed over its heads",
     "for (long n = 0; n < N; n++) g->dB[off + n] += tmp[n];", "for (long n = 0; n < N; n++) g->dB[off + n] = tmp[n];"),
]

PIN_CASES = [
    lambda o: pins.test_complex_ssm_equivalence(o),
    lambda o: pins.test_matrix_form(o),
    lambda o: pins.test_closed_form(o, 7),
    lambda o: pins.test_reduction_mamba2(o),
    lambda o: pins.test_mimo_r1_equals_siso(o),
    lambda o: pins.test_mimo_is_r2_siso_calls(o),
    lambda o: pins.test_split_schedules_siso(o, [2, 4]),
    lambda o: pins.test_chunked_equals_loop(o, 4, 37),
    lambda o: pins.test_factored_decode_from_zero_equals_mimo_loop(o, 3),
    lambda o: pins.test_mimo_decode_steps_equal_mimo_loop(o),
    lambda o: pins.test_grouped_partial_siso(o, 2, 1),
    lambda o: pins.test_partial_rope_turns_only_first_pairs(o),
    lambda o: gpins.test_siso_grad_matches_finite_differences(2),
    lambda o: gpins.test_siso_grad_norm_bias_groups_partial(),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(oracle_mod, tmp_path, name, old, new):
    src = open(oracle_mod.oracle_source_path()).read()
    assert src.count(old) >= 1, "mutation site not found: " + name
    mutated = tmp_path / "m3_oracle_mut.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = oracle_mod.compile_source(str(mutated), str(tmp_path / "libmut.so"))
    failures = 0
    with oracle_mod.use_library(lib):
        for case in PIN_CASES:
            try:
                case(oracle_mod)
            except AssertionError:
                failures += 1
    assert failures > 0, "no pin caught the planted mistake: " + name
