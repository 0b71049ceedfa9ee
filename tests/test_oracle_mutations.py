"""The pins have teeth: each test plants one plausible mistake in a copy of
the C checker (a dropped factor, a flipped sign, a transposed index, a wrong
rounding or divisor), builds it, and requires the pin aimed at that part of
the method to fail on it.  CPU only; the shipped checker is not touched."""
import os
import subprocess

import numpy as np
import pytest

import oracle.gptq as og
import test_oracle_pins as pins

# (name, text in the checker, planted replacement, pins that must fail)
MUTATIONS = [
    ("hessian drops the factor 2", "double a = 2.0 * xt[i];", "double a = xt[i];",
     [("test_hessian_matches_brute_force_triple_loop", ()), ("test_hessian_closed_form_small", ())]),
    ("compensation with the wrong sign",
     "for (int64_t k = c + 1; k < d_in; k++) w[k] -= e * U[c * d_in + k];",
     "for (int64_t k = c + 1; k < d_in; k++) w[k] += e * U[c * d_in + k];",
     [("test_two_columns_closed_form_compensation", ()), ("test_gptq_beats_rtn_on_output_error", ())]),
    ("error not divided by the pivot", "double e = (w[c] - what) / U[c * d_in + c];",
     "double e = (w[c] - what) * U[c * d_in + c];",
     [("test_error_identity_w_minus_q_equals_e_u", (False, -1, 0))]),
    ("lazy batch with a transposed factor", "acc += e_row[i] * U[i * d_in + k];",
     "acc += e_row[i] * U[k * d_in + i];",
     [("test_blocked_equals_unblocked", (32, [8, 32]))]),
    ("zero point truncated", "float z = rintf(zr);", "float z = floorf(zr);",
     [("test_quantizer_golden_cases_via_rtn_and_gptq", ())]),
    ("OBS row scaled by the pivot instead of its root",
     "for (int64_t j = c; j < d; j++) U[c * d + j] = M[c * d + j] / r;",
     "for (int64_t j = c; j < d; j++) U[c * d + j] = M[c * d + j] / p;",
     [("test_obs_upper_equals_lapack_cholesky_of_inverse", (8, 10.0))]),
    ("Q4_K offset with the wrong sign", "float qr = ((float)w[c] + o) / s;",
     "float qr = ((float)w[c] - o) / s;",
     [("test_q4k_without_compensation_picks_the_nearest_grid_point", ()),
      ("test_q4k_golden_worked_example", ())]),
    ("Q4_K super-block scale over 15 levels", "d = smax / 63.0f;", "d = smax / 15.0f;",
     [("test_q4k_super_block_scale_is_attained", ()), ("test_q4k_golden_worked_example", ())]),
    ("Q4_K without error feedback",
     "for (int64_t k = c + 1; k < b1; k++) w[k] -= e * U[c * d_in + k];\n                if (c == b1 - 1) {\n                    for (int64_t k = b1; k < d_in; k++) {\n                        double acc = 0.0;\n                        for (int64_t i = b0; i < b1; i++) acc += e_row[i] * U[i * d_in + k];\n                        w[k] -= acc;\n                    }\n                }\n            }\n        }\n        if (E) memcpy(E + r * d_in, e_row, (size_t)d_in * sizeof(double));\n        free(e_row);\n    }\n    return status;\n}\n",
     None,
     [("test_q4k_gptq_lowers_the_output_error_of_round_to_nearest", ())]),
]


def _mutant(tmp_path, old, new):
    src = open(og._SRC).read()
    if new is None:
        # the Q4_K loop only: no correction of the later columns
        head, tail = src.split("int orc_gptq_rows_q4k(", 1)
        assert tail.count("w[k] -= e * U[c * d_in + k];") == 2
        tail = tail.replace("w[k] -= e * U[c * d_in + k];", "(void)0;")
        src = head + "int orc_gptq_rows_q4k(" + tail
    else:
        assert old in src, old
        src = src.replace(old, new, 1)
    c_path = os.path.join(tmp_path, "mutant.c")
    so_path = os.path.join(tmp_path, "mutant.so")
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                           "-fno-fast-math", "-fPIC", "-shared", c_path, "-o", so_path, "-lm"])
    import ctypes
    return og.configure(ctypes.CDLL(so_path))


@pytest.mark.parametrize("name,old,new,targets", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_a_planted_mistake(tmp_path, monkeypatch, name, old, new, targets):
    og._load()                              # the shipped checker stays built
    monkeypatch.setattr(og, "_lib", _mutant(str(tmp_path), old, new))
    for pin, args in targets:
        with pytest.raises((AssertionError, ValueError, og.NotPositiveDefinite)):
            with np.errstate(all="ignore"):
                getattr(pins, pin)(*args)


def test_the_shipped_checker_passes_the_same_pins():
    for _, _, _, targets in MUTATIONS:
        for pin, args in targets:
            getattr(pins, pin)(*args)
