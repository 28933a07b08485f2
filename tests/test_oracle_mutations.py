"""Plant plausible mistakes in a copy of the oracle's C source and check that the pins catch each one.

Every mutant is compiled from a modified copy of ``oracle/kda_oracle.c`` into a temporary
directory and loaded by a child pytest run of ``test_oracle_pins.py`` through the
``KDA_ORACLE_LIB`` override; the child run must FAIL.  The unmodified source must pass.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")

# (name, exact text in kda_oracle.c, replacement)
MUTANTS = [
    ("rate outside the sigmoid", "g = lower_bound / (1.0 + exp(-rate * x));",
     "g = rate * lower_bound / (1.0 + exp(-x));"),
    ("rate inside the softplus", "const double sp = (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));\n                    g = -rate * sp;",
     "const double y = rate * x; const double sp = (y > 0.0 ? y : 0.0) + log1p(exp(-fabs(y)));\n                    g = -sp;"),
    ("dt_bias ignored", "g_raw[idx] + (dt_bias ? dt_bias[(long)h * K + d] : 0.0)", "g_raw[idx]"),
    ("decay per value column", "const double a = exp(gt[d]);\n                for (int j = 0; j < V; ++j) S[(long)d * V + j] *= a;",
     "for (int j = 0; j < V; ++j) S[(long)d * V + j] *= exp(gt[j < K ? j : K - 1]);"),
    ("predict before decay", "/* step 1 */", "/* step 1 moved */ goto step2; step1_late:"),
    ("residual sign flipped", "p[j] = vt[j] - p[j]; /* p now holds r */", "p[j] = p[j] - vt[j];"),
    ("beta dropped from the write", "const double a = bt * kt[d];", "const double a = kt[d];"),
    ("scale not applied", "for (int j = 0; j < V; ++j) ot[j] *= scale;", "(void)scale;"),
    ("read before the write", "/* step 4 */", "/* step 4 */ (void)0;"),
    ("GVA tiled instead of interleaved", "const int h = hv / G;\n        double* S = (double*)malloc(sizeof(double) * (size_t)K * V);\n        double* p",
     "const int h = hv % H;\n        double* S = (double*)malloc(sizeof(double) * (size_t)K * V);\n        double* p"),
    ("S0 ignored", "if (S0) memcpy(S, S0 + pair * (long)K * V, sizeof(double) * (size_t)K * V);\n        else memset(S, 0, sizeof(double) * (size_t)K * V);\n        for (int t = 0; t < T; ++t) {",
     "memset(S, 0, sizeof(double) * (size_t)K * V);\n        for (int t = 0; t < T; ++t) {"),
]


def _special(src, name):
    """Mutants that need more than one textual edit."""
    if name == "predict before decay":
        # move the decay after the prediction: run step 2 on S_{t-1}, then decay, then write
        a = src.index("/* step 1 */")
        b = src.index("/* step 2 */")
        c = src.index("/* step 3 */")
        step1, step2 = src[a:b], src[b:c]
        return src[:a] + step2 + step1 + src[c:]
    if name == "read before the write":
        c = src.index("/* step 3 */")
        d = src.index("/* step 4 */")
        e = src.index("if (S_out) memcpy(S_out + pair")
        # end of the token loop is the closing brace just before S_out copy
        end = src.rindex("}", d, e)
        step3, step4 = src[c:d], src[d:end]
        return src[:c] + step4 + step3 + src[end:]
    return None


def _build(tmp_path, src_text, tag):
    c = tmp_path / f"mut_{tag}.c"
    so = tmp_path / f"libmut_{tag}.so"
    c.write_text(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(so), str(c), "-lm"],
                   check=True)
    return str(so)


def _run_pins(lib):
    env = dict(os.environ, KDA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    return r.returncode


def test_unmutated_copy_passes(tmp_path):
    assert _run_pins(_build(tmp_path, open(SRC).read(), "none")) == 0


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    mutated = _special(src, name)
    if mutated is None:
        assert src.count(old) == 1, f"mutation anchor for '{name}' not found exactly once"
        mutated = src.replace(old, new)
    assert mutated != src
    assert _run_pins(_build(tmp_path, mutated, str(abs(hash(name))))) != 0, f"pins did not catch: {name}"
