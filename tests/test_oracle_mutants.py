"""The oracle pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (a dropped term, a wrong
sign, a wrong index or head map, a transposed operand), builds that copy into a
scratch directory and runs the pin suite against it in a child process.  The
pin suite has to fail for every mutant.  The real oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "norm_eps_outside_root": ("sqrt(ss / (double)D + eps)", "(sqrt(ss / (double)D) + eps)"),
    "norm_sum_not_mean": ("sqrt(ss / (double)D + eps)", "sqrt(ss + eps)"),
    "rope_sign_flip": ("yr[ib] = xa * s + xb * c;", "yr[ib] = -xa * s + xb * c;"),
    "rope_theta_exponent": ("-2.0 * (double)i / (double)D", "-1.0 * (double)i / (double)D"),
    "rope_pairing": ("int ib = interleaved ? 2 * i + 1 : i + half;",
                     "int ib = interleaved ? 2 * i + 1 : 2 * i + 1;"),
    "rope_position_offset": ("double p = (double)pos[n];", "double p = (double)pos[n] + 1.0;"),
    "head_map_modulo": ("int64_t kvh = h / g;", "int64_t kvh = h % Hkv;"),
    "causal_exclusive": ("int64_t nvis = qpos[bt] + 1;", "int64_t nvis = qpos[bt] > 0 ? qpos[bt] : 1;"),
    "scale_dropped": ("        s *= scale;\n", "\n"),
    "softmax_unnormalised": ("double p = scores[u] / l;", "double p = scores[u];"),
    "values_read_from_keys": ("const double *vr = v + ", "const double *vr = k + "),
    "bf16_shift": ("((uint32_t)bits) << 16", "((uint32_t)bits) << 15"),
    "document_mask_ignored": ("if (kdoc && kdoc[b * Tk + u] != qdoc[bt]) {", "if (0) {"),
    "document_mask_by_position": ("if (kdoc && kdoc[b * Tk + u] != qdoc[bt]) {",
                                  "if (kdoc && kdoc[b * Tk + u] != qdoc[b * Tq + u]) {"),
}


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found exactly once: %r" % old
    mut_src = tmp_path / "oracle_mut.c"
    mut_src.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", str(mut_src),
                           "-o", str(lib), "-lm"])
    env = dict(os.environ, GQA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant %s:\n%s" % (name, r.stdout[-2000:])


@pytest.mark.slow
def test_unmutated_copy_passes(tmp_path):
    """Control: the same harness on an unchanged copy must pass."""
    lib = tmp_path / "liboracle_copy.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", SRC,
                           "-o", str(lib), "-lm"])
    env = dict(os.environ, GQA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
