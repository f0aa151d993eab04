"""The oracle pins must catch plausible mistakes in the oracle's Python steps.

The companion of test_oracle_mutants.py (which plants mistakes in oracle.c):
here each case plants one mistake in a copy of oracle/__init__.py -- the
attention backward, the RoPE context-extension frequencies, the assembly of a
continuation chunk's keys -- and runs the pins that concern that step against
the copy in a child process (the copy loads the real, unmodified C oracle).
The pins have to fail for every mutant; the real oracle is never modified.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "__init__.py")

# name: (anchor, replacement, -k expression selecting the pins that concern the step)
MUTANTS = {
    "bwd_rowsum_dropped": ("dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))", "dS = P * dP",
                           "backward"),
    "bwd_dk_unscaled": ("dk[b, :, kvh] += scale * (dS.T @ Q)", "dk[b, :, kvh] += (dS.T @ Q)",
                        "backward"),
    "bwd_dv_untransposed": ("dV = P.T @ dO", "dV = P @ dO", "backward"),
    "bwd_group_overwritten": ("dv[b, :, kvh] += dV", "dv[b, :, kvh] = dV", "backward"),
    "bwd_dq_from_values": ("dq[b, :, h] = scale * (dS @ K)", "dq[b, :, h] = scale * (dS @ V)",
                           "backward"),
    "bwd_lse_without_max": ("lse[b, h] = (m + np.log(l))[:, 0]", "lse[b, h] = np.log(l)[:, 0]",
                            "backward"),
    "ntk_exponent": ("base = base * s ** (D / (D - 2.0))", "base = base * s ** (D / (D - 1.0))",
                     "ntk or scaling or scaled"),
    "linear_multiplies": ("return theta / s", "return theta * s",
                          "linear or scaling or scaled"),
    "yarn_ramp_reversed": ("return (1.0 - ramp) * theta / s + ramp * theta",
                           "return ramp * theta / s + (1.0 - ramp) * theta", "yarn or scaling"),
    "yarn_turns_without_2pi": ("turns = self.original_max_pos * theta / (2.0 * math.pi)",
                               "turns = self.original_max_pos * theta", "yarn"),
    "yarn_temperature": ("0.1 * math.log(self.factor) + 1.0", "0.2 * math.log(self.factor) + 1.0",
                         "yarn"),
    "chunk_prefix_dropped": ("keys[b, :P] = kc[b, :, :P].transpose(1, 0, 2)", "keys[b, :P] = 0.0",
                             "chunk"),
    "chunk_values_from_keys": ("vals[b, P:P + n] = v[b, :n]", "vals[b, P:P + n] = k[b, :n]",
                               "chunk"),
}


def _tree(root, src_text):
    """A scratch project: the pins, the golden fixtures, the package (linked) and
    an oracle package whose Python part is src_text."""
    shutil.copytree(HERE, os.path.join(root, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(root, "oracle"))
    with open(os.path.join(root, "oracle", "__init__.py"), "w") as f:
        f.write(src_text)
    shutil.copy(os.path.join(ROOT, "oracle", "oracle.c"), os.path.join(root, "oracle", "oracle.c"))
    os.symlink(os.path.join(ROOT, "rope_gqa_kv_b200"), os.path.join(root, "rope_gqa_kv_b200"))


def _run(name, scratch, lib):
    """Run the selected pins against a copy of the oracle's Python part, mutated
    unless name is None; returns the child's (returncode, stdout tail)."""
    src = open(SRC).read()
    if name is None:
        select = " or ".join(sorted({m[2] for m in MUTANTS.values()}))
    else:
        old, new, select = MUTANTS[name]
        if src.count(old) != 1:
            return None, "mutation anchor not found exactly once: %r" % old
        src = src.replace(old, new)
    root = os.path.join(scratch, name or "control")
    _tree(root, src)
    env = dict(os.environ, GQA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-k", select, os.path.join(root, "tests", "test_oracle_pins.py")],
                       cwd=root, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:] + r.stderr[-1000:]


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    """Every mutant and the control, run side by side (one child per case)."""
    import oracle
    lib = oracle.build()
    scratch = str(tmp_path_factory.mktemp("oracle_py_mutants"))
    names = sorted(MUTANTS) + [None]
    workers = max(2, min(len(names), (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        return dict(zip(names, ex.map(lambda n: _run(n, scratch, lib), names)))


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_python_mutant(name, results):
    rc, out = results[name]
    assert rc is not None, out
    assert "passed" in out or "failed" in out, out
    assert rc != 0, "pins did not catch mutant %s:\n%s" % (name, out)


@pytest.mark.slow
def test_unmutated_python_copy_passes(results):
    """Control: the same harness on an unchanged copy passes every selected pin."""
    rc, out = results[None]
    assert rc == 0, out
    assert " passed" in out
