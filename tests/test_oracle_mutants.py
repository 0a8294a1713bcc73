"""Each plausible mistake planted in a copy of the C oracle must make at
least one pin fail.  The mutants are built on the CPU from a patched copy of
``oracle/kda_oracle.c`` in a temporary directory; the committed oracle is
never modified."""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("no_decay", "alpha[i] = exp(gi);", "alpha[i] = 1.0;"),
    ("decay_sign", "alpha[i] = exp(gi);", "alpha[i] = exp(-gi);"),
    ("no_floor", "gt[i] > g_floor ? gt[i] : g_floor", "gt[i]"),
    ("decay_on_columns", "S[(size_t)i * dv + j] *= alpha[i];", "S[(size_t)i * dv + j] *= alpha[j];"),
    ("erase_sign", "(vt[j] - u[j])", "(vt[j] + u[j])"),
    ("no_erase", "bt * kt[i] * (vt[j] - u[j])", "bt * kt[i] * vt[j]"),
    ("no_beta_on_write", "bt * kt[i] * (vt[j] - u[j])", "kt[i] * (vt[j] - u[j])"),
    ("recall_before_decay", "u[j] += S[(size_t)i * dv + j] * kt[i];",
     "u[j] += S[(size_t)i * dv + j] * kt[i] / alpha[i];"),
    ("transposed_readout", "ot[j] += S[(size_t)i * dv + j] * qt[i];",
     "ot[j] += S[(size_t)j * dv + i] * qt[i];"),
    ("readout_with_key", "ot[j] += S[(size_t)i * dv + j] * qt[i];",
     "ot[j] += S[(size_t)i * dv + j] * kt[i];"),
    ("no_scale", "ot[j] *= scale;", "ot[j] *= 1.0;"),
    ("gate_sign", "exp(-gate[rv + j])", "exp(gate[rv + j])"),
    ("ignore_S0", "if (S0)\n", "if (0)\n"),
    ("off_by_one_head", "((size_t)t * H + h) * dk;", "((size_t)t * H + (h + 1) % H) * dk;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor missing: {old!r}"
    mut_src = tmp_path / f"mut_{name}.c"
    mut_src.write_text(src.replace(old, new, 1))
    so = str(tmp_path / f"libmut_{name}.so")
    import subprocess
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                    str(mut_src), "-o", so, "-lm"], check=True)
    lib = oracle._load(so)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
