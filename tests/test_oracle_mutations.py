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


# ---------------------------------------------------------------------------
# The Python-level oracle functions (segment maps, composition, projections,
# I/O rounding): each mutant replaces one function with a plausible mistake
# and one of the pins in tests/test_oracle_pins.py must fail.
# ---------------------------------------------------------------------------

def _mut_compose_reversed(orig):
    return lambda P, S, x0=None, reverse=False: orig(P, S, x0, not reverse)


def _mut_compose_swapped(orig):
    import numpy as np

    def f(P, S, x0=None, reverse=False):
        P = np.asarray(P, dtype=np.float64)
        S = np.asarray(S, dtype=np.float64)
        x = np.zeros(P.shape[1:]) if x0 is None else np.array(x0, dtype=np.float64)
        for j in (range(P.shape[0] - 1, -1, -1) if reverse else range(P.shape[0])):
            x = S[j] * x + P[j]
        return x
    return f


def _mut_project_order(orig):
    def f(x, W, io_dtype):
        a, v, q = orig(x, W, io_dtype)
        return v, a, q
    return f


def _mut_round_bf16_truncates(orig):
    import numpy as np

    def f(x, io_dtype):
        if io_dtype != "bf16":
            return orig(x, io_dtype)
        u = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32)).view(np.uint32)
        return (u >> 16 << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    return f


def _mut_scan_map_short_product(orig):
    import numpy as np

    def f(a, v, mode):
        P, S = orig(a, v, mode)
        a = np.asarray(a, dtype=np.float64)
        return np.prod(1.0 / (1.0 + np.exp(-a[:, :-1])), axis=1), S
    return f


def _mut_bwd_map_ignores_E_init(orig):
    return lambda a, v, q, dy, mode, E_init=None: orig(a, v, q, dy, mode, E_init=None)


def _mut_output_projection_transposed(orig):
    import numpy as np
    return lambda y, W_O, io_dtype: orig(y, np.asarray(W_O, dtype=np.float64).T, io_dtype)


def _mut_output_projection_unrounded_input(orig):
    import numpy as np
    import oracle

    def f(y, W_O, io_dtype):
        y = np.asarray(y, dtype=np.float64)
        return oracle.round_io(y.reshape(y.shape[0], y.shape[1], -1) @ np.asarray(W_O, dtype=np.float64).T, io_dtype)
    return f


def _mut_output_projection_unrounded_output(orig):
    import numpy as np
    import oracle

    def f(y, W_O, io_dtype):
        y = oracle.round_io(np.asarray(y, dtype=np.float64), io_dtype)
        return y.reshape(y.shape[0], y.shape[1], -1) @ np.asarray(W_O, dtype=np.float64).T
    return f


PY_MUTANTS = [
    ("compose_order_reversed", "compose", _mut_compose_reversed, "test_compose_order_small_example", ()),
    ("compose_P_S_swapped", "compose", _mut_compose_swapped, "test_compose_order_small_example", ()),
    ("project_order_swapped", "project", _mut_project_order, "test_project_hand_example", ()),
    ("round_bf16_truncates", "round_io", _mut_round_bf16_truncates, "test_round_io_matches_torch_conversions", ()),
    ("scan_map_drops_last_gate", "scan_map", _mut_scan_map_short_product,
     "test_scan_map_is_the_affine_map_of_the_slice", (1,)),
    ("bwd_map_ignores_E_init", "scan_bwd_map", _mut_bwd_map_ignores_E_init,
     "test_scan_bwd_map_is_the_affine_map_of_the_slice", (1,)),
    ("output_projection_transposed", "output_projection", _mut_output_projection_transposed,
     "test_output_projection_hand_example_and_special_cases", ()),
    ("output_projection_unrounded_input", "output_projection", _mut_output_projection_unrounded_input,
     "test_output_projection_rounds_its_input_and_its_output", ()),
    ("output_projection_unrounded_output", "output_projection", _mut_output_projection_unrounded_output,
     "test_output_projection_rounds_its_input_and_its_output", ()),
]


@pytest.mark.parametrize("name,fn,make,pin,args", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_pins_catch_python_mutant(monkeypatch, name, fn, make, pin, args):
    import oracle
    from tests import test_oracle_pins as pins
    getattr(pins, pin)(*args)                       # the pin passes on the real oracle
    monkeypatch.setattr(oracle, fn, make(getattr(oracle, fn)))
    with pytest.raises(AssertionError):
        getattr(pins, pin)(*args)
