"""The oracle's pins catch plausible mistakes: each case plants one mistake in a
copy of the oracle's C source, a dropped term, a wrong sign, or a wrong operand
or factor, builds it, and runs the pin tests (tests/test_oracle.py) against that
build in a subprocess.  The case passes only if some pin fails.  An unaltered
copy built the same way passes every pin.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sf_oracle.c")

# (text in sf_oracle.c, replacement, what the mistake is); the first occurrence is replaced
MUTATIONS = [
    ("S[i * dv + j] = a * (S[i * dv + j] - bt * kt[i] * y[j]) + bt * kt[i] * vt[j];",
     "S[i * dv + j] = a * (S[i * dv + j] - bt * kt[i] * y[j]) + kt[i] * vt[j];",
     "delta-rule write without beta"),
    ("S[i * dv + j] = a * (S[i * dv + j] - bt * kt[i] * y[j]) + bt * kt[i] * vt[j];",
     "S[i * dv + j] = a * S[i * dv + j] - bt * kt[i] * y[j] + bt * kt[i] * vt[j];",
     "decay applied to the old state only"),
    ("for (int j = 0; j < dv; ++j) S[i * dv + j] = a * S[i * dv + j] + kt[i] * vt[j];",
     "for (int j = 0; j < dv; ++j) S[i * dv + j] = S[i * dv + j] + kt[i] * vt[j];",
     "linear attention without its decay"),
    ("for (int j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qt[i];",
     "for (int j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * kt[i];",
     "output read with the key"),
    ("const double a = g ? exp(g[ti]) : 1.0;", "const double a = g ? exp(-g[ti]) : 1.0;",
     "gate sign (forward)"),
    ("dkt[i] += -bt * acc;", "dkt[i] += bt * acc;", "sign of the delta term of dk"),
    ("acc += dX[i * dv + j] * y[j] + P[i * dv + j] * z[j];", "acc += dX[i * dv + j] * y[j];",
     "dk without the P z term"),
    ("for (int j = 0; j < dv; ++j) db -= y[j] * z[j];", "for (int j = 0; j < dv; ++j) db += 0;",
     "dbeta without the -y^T z term"),
    ("if (g) dg[ti] = a * da;", "if (g) dg[ti] = da;", "dg without the factor a"),
    ("dS[i * dv + j] = dX[i * dv + j] - bt * kt[i] * z[j];", "dS[i * dv + j] = dX[i * dv + j];",
     "state gradient without the -b k z^T term"),
    ("dS[i * dv + j] *= a;", "dS[i * dv + j] *= 1.0;", "linear-attention state gradient not decayed"),
    ("for (int j = 0; j < dv; ++j) dS[i * dv + j] += qt[i] * dot[j];",
     "for (int j = 0; j < dv; ++j) dS[i * dv + j] += kt[i] * dot[j];", "read-out gradient with the key"),
    ("for (int j = 0; j < dv; ++j) dvt[j] *= bt;", "for (int j = 0; j < dv; ++j) dvt[j] *= 1.0;",
     "delta-rule dv without beta"),
    ("dkt[i] = acc;", "dkt[i] = -acc;", "linear-attention dk sign"),
]


def _run_pins(tmp_path, source: str):
    src = tmp_path / "sf_oracle.c"
    src.write_text(source)
    lib = tmp_path / "libsf_oracle_variant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", str(src), "-o",
                           str(lib), "-lm"])
    env = dict(os.environ, SF_ORACLE_LIB=str(lib))
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"),
                           "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_unaltered_copy_passes_the_pins(tmp_path):
    r = _run_pins(tmp_path, open(SRC).read())
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("frm,to,what", MUTATIONS, ids=[m[2] for m in MUTATIONS])
def test_pins_catch_a_planted_mistake(tmp_path, frm, to, what):
    source = open(SRC).read()
    assert frm in source, f"mutation target not found: {frm}"
    r = _run_pins(tmp_path, source.replace(frm, to, 1))
    assert r.returncode == 1, f"no pin caught: {what}\n{r.stdout[-2000:]}"
