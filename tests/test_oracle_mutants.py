"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle into a temporary directory, plants one mistake in
the copied C source (on the CPU, never in the product), rebuilds it there and
runs ``tests/test_oracle.py`` against the copy.  The run must fail.  A
forward site that the backward's recomputation shares is mutated in both;
the ``bwd_`` sites exist in the backward adjoint only.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "write_sign": ("row[j] += kc * u[j];", "row[j] -= kc * u[j];"),
    "beta_dropped": ("u[j] = bt * (vt[j] - u[j]);", "u[j] = (vt[j] - u[j]);"),
    "decay_dropped": ("const double a = exp(gt[c]);", "const double a = 1.0;"),
    "decay_doubled": ("const double a = exp(gt[c]);", "const double a = exp(2.0 * gt[c]);"),
    "scale_dropped": ("ot[j] = scale * o[j];", "ot[j] = o[j];"),
    "key_for_query": ("const double qc = qt[c];", "const double qc = kt[c];"),
    # the backward adjoint
    "bwd_erase_sign": ("drow[j] -= bt * kt[c] * du[j];", "drow[j] += bt * kt[c] * du[j];"),
    "bwd_decay_dropped": ("for (int64_t j = 0; j < dv; ++j) drow[j] *= a;", ""),
    "bwd_dg_undecayed": ("gacc += drow[j] * sb;", "gacc += drow[j] * row[j];"),
    "bwd_dbeta_from_u": ("db += du[j] * r[j];", "db += du[j] * u[j];"),
    "bwd_dk_erase_dropped": ("dkt[c] -= bt * acc;", "dkt[c] -= 0.0 * acc;"),
    "bwd_dq_scale_dropped": ("dqt[c] = scale * acc;", "dqt[c] = acc;"),
    "bwd_output_adjoint_q_for_k": ("drow[j] += scale * qt[c] * dot[j];",
                                   "drow[j] += scale * kt[c] * dot[j];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    before, after = MUTANTS[name]
    src_path = os.path.join(ROOT, "oracle", "kda_oracle.c")
    src = open(src_path).read()
    assert before in src, f"mutation site for {name} not found"
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (tmp_path / "oracle" / "kda_oracle.c").write_text(src.replace(before, after))
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle.py"], cwd=tmp_path, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout
