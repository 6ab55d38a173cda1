"""Plant plausible mistakes in copies of the oracle and check that the pins
in ``test_oracle.py`` catch every one of them.

Each mutant is a copy of ``oracle/ssd_oracle.c`` with one edit (a dropped
term, a wrong sign or index, a transposed operand), compiled on the CPU; the
pin suite is then re-run against it in a child pytest process and must fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ssd_oracle.c")

MUTANTS = {
    "no_decay": ("hp[n] = a * hp[n] + u * Bt[n];", "hp[n] = hp[n] + u * Bt[n];"),
    "no_dt_on_input": ("const double u = d * xt[p];", "const double u = xt[p];"),
    "readout_before_update": (
        "hp[n] = a * hp[n] + u * Bt[n];\n                acc += hp[n] * Ct[n];",
        "acc += hp[n] * Ct[n];\n                hp[n] = a * hp[n] + u * Bt[n];"),
    "wrong_group_index": ("    const int g = h / (H / G);\n    const double Dh = D ? D[h] : 0.0;\n    if (init_state)",
                          "    const int g = h % G;\n    const double Dh = D ? D[h] : 0.0;\n    if (init_state)"),
    "no_skip_term": ("yt[p] = acc + Dh * xt[p];", "yt[p] = acc;"),
    "decay_sign": ("const double a = exp(d * A[h]);\n        const double* xt = x + (((size_t)b * L + t) * H + h) * P;",
                   "const double a = exp(-d * A[h]);\n        const double* xt = x + (((size_t)b * L + t) * H + h) * P;"),
    "mask_off_by_one": ("for (int k = i + 1; k <= j; ++k)", "for (int k = i; k <= j; ++k)"),
    "mask_transposed": ("const double m = Lm[(size_t)j * L + i]", "const double m = Lm[(size_t)i * L + j]"),
    "step_no_dt": ("*hv = a * *hv + d * xt[p] * Bt[n];", "*hv = a * *hv + xt[p] * Bt[n];"),
    "step_decay_sign": ("const double a = exp(d * A[h]);\n            const double Dh",
                        "const double a = exp(-d * A[h]);\n            const double Dh"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path, oracle):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not unique"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(text.replace(old, new))
    lib = oracle.compile_source(str(mut_src), str(tmp_path / "libmutant.so"))
    env = dict(os.environ, SSD_ORACLE_MUTANT_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
