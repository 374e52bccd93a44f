"""The oracle's pins catch plausible mistakes.

Each case copies the oracle's C source into a temporary directory, plants one
mistake (a flipped sign, a dropped term, a wrong operand, a skipped
transpose), compiles it, loads it in place of the real oracle and runs the
pin that should reject it.  The real oracle is never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_adamw as adamw
import test_oracle_lite as lite
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "muon_oracle.c")

MUTATIONS = [
    # (name, original text, planted text, pin functions that must fail)
    ("drop_c_term", "B[i] = b * A[i] + c * AA[i];", "B[i] = b * A[i];",
     [lambda: pins.test_ns_poly_closed_form_through_svd((16, 40))]),
    ("update_sign", "X[i] = a * X[i] + BX[i];", "X[i] = a * X[i] - BX[i];",
     [lambda: pins.test_ns_poly_closed_form_through_svd((16, 40))]),
    ("gram_not_aat", "mat_mul_aat(X, A, s, l);          /* A = X X^T      */",
     "mat_mul(X, X, A, s, s, s);", [lambda: pins.test_ns_poly_closed_form_through_svd((8, 8))]),
    ("mona_difference_sign", "double D = G[i] - Gp[i];", "double D = Gp[i] - G[i];",
     [pins.test_mona_hand_example]),
    ("mona_uses_old_buffer", "(1.0 - beta_a) * D;\n        double Gt = G[i] + alpha * An;",
     "(1.0 - beta_a) * D;\n        double Gt = G[i] + alpha * A[i];",
     [pins.test_mona_hand_example]),
    ("decay_sign", "W[i] = W[i] - eta * (gamma * O[i] + lambda * W[i]);",
     "W[i] = W[i] - eta * (gamma * O[i] - lambda * W[i]);", [pins.test_weight_update_hand_example]),
    ("gram_R_update_missing_h", "mat_mul(T, H, R, s, s, s);", "memcpy(R, T, sizeof(double) * ss);",
     [lambda: pins.test_gram_route_equals_direct_route_in_exact_arithmetic((0, 9), "converged")]),
    ("gram_restart_no_divide", "X[i] = Xn[i] / f;", "X[i] = Xn[i];",
     [lambda: pins.test_gram_route_equals_direct_route_in_exact_arithmetic((0, 2, 4), "quintic6")]),
    ("jacobi_rotation_sign", "xq[j] = sn * a + c * b;", "xq[j] = -sn * a + c * b;",
     [lambda: pins.test_polar_matches_lapack_svd((16, 32))]),
    ("orientation_not_transposed_back", "else transpose(X, O, cols, rows);",
     "else memcpy(O, X, sizeof(double) * sl);", [pins.test_orthogonalise_orientation_and_scale]),
    ("lite_b_update_sign", "double Bn = beta_a * An - (1.0 - beta_a) * G[i];",
     "double Bn = beta_a * An + (1.0 - beta_a) * G[i];", [lite.test_mona_lite_hand_example]),
    ("lite_difference_weight", "double An = B[i] + (1.0 - beta_a) * G[i];",
     "double An = B[i] + beta_a * G[i];",
     [lambda: lite.test_mona_lite_equals_mona_without_rounding(0.9, 0.5, 0.95)]),
    ("adamw_bias_correction_step", "const double c1 = 1.0 - pow(b1, (double)t);",
     "const double c1 = 1.0 - pow(b1, (double)(t + 1));", [adamw.test_adamw_hand_example_two_steps]),
    ("adamw_no_sqrt", "const double upd = (mn / c1) / (sqrt(vn / c2) + eps);",
     "const double upd = (mn / c1) / ((vn / c2) + eps);", [adamw.test_adamw_hand_example_two_steps]),
    ("adamw_coupled_decay", "W[i] = W[i] - lr * (upd + wd * W[i]);", "W[i] = W[i] - lr * upd;",
     [adamw.test_adamw_zero_gradient_is_pure_decay]),
    ("bf16_precision", "return round_to_format(x, 8, -126, 0x1.fep127);",
     "return round_to_format(x, 7, -126, 0x1.fep127);",
     [pins.test_round_bf16_matches_torch_on_float32_values]),
]


@pytest.mark.parametrize("name,orig,planted,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_rejects_planted_mistake(tmp_path, name, orig, planted, checks):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not unique"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(orig, planted))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           "-ffp-contract=off", "-o", str(so), str(mut), "-lm"])
    saved = oracle._lib
    oracle._lib = oracle.configure(ctypes.CDLL(str(so)))
    try:
        for check in checks:
            with pytest.raises((AssertionError, RuntimeError)):
                check()
    finally:
        oracle._lib = saved
