"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake (a dropped term, a wrong sign, an
off-by-one time index, a wrong constant) in a private copy of the oracle's C
source, builds it into a temporary library, and runs the pin suite against
that build in a subprocess.  The pin suite must fail for every mutant.
Nothing here touches a GPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "esa_oracle.c")

# (name, original text, planted text, which occurrence: None = all)
MUTANTS = [
    ("eps_value", "#define ESA_ORACLE_EPS 1e-6", "#define ESA_ORACLE_EPS 1e-5", None),
    ("eps_outside_sqrt", "1.0 / sqrt(sumsq / (double)D + ESA_ORACLE_EPS)",
     "1.0 / (sqrt(sumsq / (double)D) + ESA_ORACLE_EPS)", None),
    ("sum_not_mean", "sumsq / (double)D + ESA_ORACLE_EPS", "sumsq + ESA_ORACLE_EPS", 0),
    ("sigmoid_neg_branch", "return e / (1.0 + e);", "return 1.0 / (1.0 + e);", None),
    ("controlled_write_dropped", "(1.0 - A) * v[i]", "v[i]", 0),
    ("e_init_ignored", "e[d] = E_init ? E_init[at_bhd(b, h, d, H, D)] : 0.0;", "e[d] = 0.0;", None),
    ("step_write_term", "(1.0 - A) * v_t[row + d]", "(1.0 + A) * v_t[row + d]", None),
    ("bwd_replay_write_term", "(1.0 - A) * v[i]", "A * v[i]", 1),
    ("bwd_prev_off_by_one", "double prev = (t == 0) ? e0[d] : Es[(size_t)(t - 1) * nd + (size_t)d];\n"
     "                    double G", "double prev = Es[(size_t)t * nd + (size_t)d];\n"
     "                    double G", None),
    ("bwd_controlled_da_drops_v", "dA = G * (prev - v[row + d]);", "dA = G * prev;", None),
    ("bwd_sigmoid_derivative", "da[row + d] = dA * A * (1.0 - A);", "da[row + d] = dA * A;", None),
    ("bwd_carry_no_gate", "hin[d] = A * G;", "hin[d] = G;", None),
    ("bwd_norm_projection_dropped", "gh[d] = r * (dn - n * dot / (double)D);", "gh[d] = r * dn;", None),
    ("bwd_dq_unnormalised", "dq[row + d] = dy[row + d] * n;", "dq[row + d] = dy[row + d] * Et[d];", None),
    ("bwd_controlled_dv", "dv[row + d] = G * (1.0 - A);", "dv[row + d] = G * A;", None),
    ("bwd_dE_final_ignored", "hin[d] = dE_final ? dE_final[at_bhd(b, h, d, H, D)] : 0.0;",
     "hin[d] = 0.0;", None),
]


def _mutate(src, old, new, which):
    if which is None:
        assert old in src, old
        return src.replace(old, new)
    parts = src.split(old)
    assert len(parts) > which + 1, (old, which)
    return old.join(parts[: which + 1]) + new + old.join(parts[which + 1:])


@pytest.mark.parametrize("name,old,new,which", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new, which):
    src = open(SRC).read()
    mutated = _mutate(src, old, new, which)
    assert mutated != src
    c_path = tmp_path / "mutant.c"
    c_path.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                    str(c_path), "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, ESA_ORACLE_LIB_OVERRIDE=str(lib))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"mutant {name} survived the pins:\n{res.stdout[-2000:]}"
