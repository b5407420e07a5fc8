"""The oracle's pins reject plausible mistakes (CPU only).

Each case copies eqat_oracle.c, plants one mistake by a textual substitution,
builds the copy with the oracle's own flags into a temporary directory and runs
the pin suite against it (EQAT_ORACLE_LIB).  The suite must fail for every
mutant; the unmodified source must pass (covered by test_oracle_pins.py).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "eqat_oracle.c")

MUTANTS = {
    "ds_drops_mask_u_term": ("const double dwds = (double)(c - zr) - (inside ? (double)u : 0.0);",
                             "const double dwds = (double)(c - zr);"),
    "ds_wrong_sign": ("const double dwds = (double)(c - zr) - (inside ? (double)u : 0.0);",
                      "const double dwds = (double)(zr - c) + (inside ? (double)u : 0.0);"),
    "dz_wrong_sign": ("acc_z += g * (double)sc * (double)(inside - 1);",
                      "acc_z += g * (double)sc * (double)(1 - inside);"),
    "clamp_bounds_exclusive": ("const int inside = (q >= 0.0f) && (q <= Q);\n                const double g",
                               "const int inside = (q > 0.0f) && (q < Q);\n                const double g"),
    "reciprocal_instead_of_division": ("const float u = w / sc;", "const float u = w * (1.0f / sc);"),
    "zero_point_not_rounded": ("const float zr = rintf(z[gi]);\n            const float w",
                               "const float zr = z[gi];\n            const float w"),
    "pack_big_endian_in_byte": ("const int shift = bits * (int)(k % per_byte);\n                packed",
                                "const int shift = bits * (per_byte - 1 - (int)(k % per_byte));\n                packed"),
    "init_divides_by_2N": ("float sc = range / Q;", "float sc = range / (Q + 1.0f);"),
    "init_zero_point_sign": ("float neg = -xmin;", "float neg = xmin;"),
    "dx_transposed_operand": ("out[k] += g * (double)What[n * K + k];",
                              "out[k] += g * (double)What[(k % N) * K + (n % K)];"),
    "round_half_away": ("const float r = rintf(u);", "const float r = roundf(u);"),
    "clamp_pass_drops_u_term": ("acc_s += g * ((double)(c - zr) - (double)u);",
                                "acc_s += g * (double)(c - zr);"),
    "clamp_pass_masks_dw": ("if (dW) dW[r * K + k] = g;",
                            "if (dW) dW[r * K + k] = (c == rintf(u) + zr) ? g : 0.0;"),
    "e2e_dz_wrong_sign": ("dz[r * G + j] = -(double)s[n * G + j] * acc;",
                          "dz[r * G + j] = (double)s[n * G + j] * acc;"),
    "e2e_dz_drops_scale": ("dz[r * G + j] = -(double)s[n * G + j] * acc;", "dz[r * G + j] = -acc;"),
    "adamw_bias_correction_outside_sqrt": ("pi -= lr * ((double)m32 / bc1) / (sqrt((double)v32 / bc2) + eps);",
                                           "pi -= lr * ((double)m32 / bc1) / (sqrt((double)v32) / bc2 + eps);"),
    "adamw_without_decoupled_decay": ("double pi = (double)p[i] * (1.0 - lr * wd);", "double pi = (double)p[i];"),
    "e2e_ds_ignores_zero_point": ("const double diff = (double)orc_code_at(packed, K, bits, n, k) - (double)zq[n * G + j];",
                                  "const double diff = (double)orc_code_at(packed, K, bits, n, k);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name, tmp_path):
    import oracle
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new)
    csrc = tmp_path / "mutant.c"
    csrc.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(csrc), "-o", str(lib), "-lm"])
    env = dict(os.environ, EQAT_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins accepted mutant {name}:\n{r.stdout[-2000:]}"
