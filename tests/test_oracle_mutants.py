"""The oracle pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (a dropped term, a wrong
sign, a wrong index or head map, a transposed operand), builds that copy into a
scratch directory and runs the pin suite against it in a child process.  The
pin suite has to fail for every mutant.  The real oracle is never modified.
"""
import concurrent.futures
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


def _run(name, scratch):
    """Build the copy of oracle.c (mutated unless name is None) and run the pins
    against it; returns the child's (returncode, stdout tail)."""
    src = open(SRC).read()
    if name is not None:
        old, new = MUTANTS[name]
        if src.count(old) != 1:
            return None, "mutation anchor not found exactly once: %r" % old
        src = src.replace(old, new)
    d = os.path.join(scratch, name or "control")
    os.makedirs(d)
    mut_src = os.path.join(d, "oracle_mut.c")
    with open(mut_src, "w") as f:
        f.write(src)
    lib = os.path.join(d, "liboracle_mut.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", mut_src, "-o", lib,
                           "-lm"])
    env = dict(os.environ, GQA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    """Every mutant and the control, run side by side (one child per case)."""
    scratch = str(tmp_path_factory.mktemp("oracle_mutants"))
    names = sorted(MUTANTS) + [None]
    workers = max(2, min(len(names), (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        return dict(zip(names, ex.map(lambda n: _run(n, scratch), names)))


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, results):
    rc, out = results[name]
    assert rc is not None, out
    assert "passed" in out or "failed" in out, out
    assert rc != 0, "pins did not catch mutant %s:\n%s" % (name, out)


@pytest.mark.slow
def test_unmutated_copy_passes(results):
    """Control: the same harness on an unchanged copy must pass."""
    rc, out = results[None]
    assert rc == 0, out
