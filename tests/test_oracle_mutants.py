"""Plant plausible mistakes in copies of the oracle source and check that the pin
suite catches every one of them (CPU only; the real oracle is untouched)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ternmoe_oracle.c")

MUTANTS = {
    "code_01_is_minus": ("case 1: return 1;", "case 1: return -1;"),
    "big_endian_in_byte": ("(row[k / 4] >> (2 * (k % 4)))", "(row[k / 4] >> (2 * (3 - k % 4)))"),
    "dropped_minus_term": ("return plus - minus;", "return plus;"),
    "ties_to_higher_index": ("l[e] > l[best]", "l[e] >= l[best]"),
    "gates_not_renormalised": ("gates[t * k + i] = ev[i] / z;", "gates[t * k + i] = ev[i];"),
    "silu_dropped": ("return g / (1.0 + exp(-g)) * u;", "return g * u;"),
    "down_scale_dropped": ("tern_dot_f64(drow, hd, f, &bad, &unchecked) * (double)sd",
                           "tern_dot_f64(drow, hd, f, &bad, &unchecked)"),
    "rms_sum_not_mean": ("sqrt(ss / (double)d + eps)", "sqrt(ss + eps)"),
    "rms_eps_outside_root": ("sqrt(ss / (double)d + eps)", "sqrt(ss / (double)d) + eps"),
    "residual_unrounded_ffn": ("bad += or_moe_ffn(L, n, T, act, y, y64, tr, NULL, NULL, NULL);\n    for (int64_t i = 0; i < T * d; i++) x_out[i] = f64_to_bf16(bf16_to_f64(x[i]) + bf16_to_f64(y[i]));",
                               "double *yy = (double *)malloc(sizeof(double) * (size_t)(T * d));\n    bad += or_moe_ffn(L, n, T, act, y, yy, tr, NULL, NULL, NULL);\n    for (int64_t i = 0; i < T * d; i++) x_out[i] = f64_to_bf16(bf16_to_f64(x[i]) + yy[i]);\n    if (y64) memcpy(y64, yy, sizeof(double) * (size_t)(T * d));\n    free(yy);"),
    "quant_truncates": ("float r = rintf(p);", "float r = truncf(p);"),
    "residual_dropped": ("f64_to_bf16(bf16_to_f64(x[i]) + bf16_to_f64(y[i]))", "y[i]"),
    "gate_up_swapped": ("h[j] = (float)silu_times(g, u);", "h[j] = (float)silu_times(u, g);"),
    "int8_scale_order": ("g = g * sg;\n                    g = g * sx;", "g = g * sx;\n                    g = g * sx;"),
    "base3_big_endian": ("value += digit * place;\n                place *= 3;",
                         "value = value * 3 + digit;\n                place *= 3;"),
    "base3_digits_swapped": ("if (v == 1) digit = 1;\n                    else if (v == -1) digit = 2;",
                             "if (v == 1) digit = 2;\n                    else if (v == -1) digit = 1;"),
}


def test_pins_pass_on_the_oracle_built_the_same_way(tmp_path):
    """Control: the unmutated source, built and loaded exactly as the mutants are, passes."""
    so = tmp_path / "orig.so"
    subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-o", str(so), SRC, "-lm"])
    env = dict(os.environ, TERNMOE_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation site vanished: " + name
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-o", str(so), str(mut), "-lm"])
    env = dict(os.environ, TERNMOE_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant " + name + "\n" + r.stdout[-2000:]


# The same for the approximate-head oracle (plain numpy): each planted mistake must fail one of
# its pins in tests/test_oracle_flashhead.py.
FH_SRC = os.path.join(ROOT, "oracle", "flashhead.py")
FH_MUTANTS = {
    "mean_off_by_one": (".sum(axis=1) / cluster_size", ".sum(axis=1) / (cluster_size - 1)"),
    "int4_scale_over_8": ("scale = absmax / 7.0", "scale = absmax / 8.0"),
    "int4_ties_away_from_zero": ("np.rint(C[nz] / scale[nz, None])", "np.trunc(C[nz] / scale[nz, None] + np.copysign(0.5, C[nz]))"),
    "nibbles_swapped": ("return (lo | (hi << 4)).astype(np.uint8)", "return (hi | (lo << 4)).astype(np.uint8)"),
    "score_scale_dropped": ("return (q @ x) * np.asarray(scale, dtype=np.float64)", "return q @ x"),
    "clusters_ties_to_higher": ("order = np.lexsort((np.arange(sc.size), -sc))", "order = np.lexsort((-np.arange(sc.size), -sc))"),
    "cluster_rows_misplaced": ("[:, None] * cluster_size + np.arange(cluster_size)", "[:, None] * (cluster_size - 1) + np.arange(cluster_size)"),
    "best_ties_to_higher": ("order = np.lexsort((ids, -logits))", "order = np.lexsort((-ids, -logits))"),
}


def test_flashhead_pins_pass_on_the_oracle_loaded_the_same_way():
    """Control: the unmutated module, loaded exactly as the mutants are, passes."""
    env = dict(os.environ, TERNMOE_FLASHHEAD_SRC=FH_SRC)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_flashhead.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(FH_MUTANTS))
def test_flashhead_pins_catch_mutant(name, tmp_path):
    old, new = FH_MUTANTS[name]
    src = open(FH_SRC).read()
    assert src.count(old) == 1, "mutation site vanished: " + name
    mut = tmp_path / "flashhead_mut.py"
    mut.write_text(src.replace(old, new))
    env = dict(os.environ, TERNMOE_FLASHHEAD_SRC=str(mut))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_flashhead.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant " + name + "\n" + r.stdout[-2000:]
