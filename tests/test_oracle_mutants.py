"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch every one of them.  The real ssd_oracle.c is never modified:
each mutant is a textual edit of a copy compiled into a temporary directory."""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")

# (name, exact text in ssd_oracle.c, replacement)
MUTANTS = [
    ("input_decayed_by_own_step", "Sp[n] = a * Sp[n] + u * Bt[n];",
     "Sp[n] = a * (Sp[n] + u * Bt[n]);"),
    ("missing_skip_term", "yt[p] = acc + D[h] * xt[p];", "yt[p] = acc;"),
    ("readout_uses_B", "u * Bt[n];\n                acc += Sp[n] * Ct[n];",
     "u * Bt[n];\n                acc += Sp[n] * Bt[n];"),
    ("readout_before_update", "Sp[n] = a * Sp[n] + u * Bt[n];\n                acc += Sp[n] * Ct[n];",
     "acc += Sp[n] * Ct[n];\n                Sp[n] = a * Sp[n] + u * Bt[n];"),
    ("interleaved_group_map", "const int64_t g = h * G / nheads;", "const int64_t g = h % G;"),
    ("input_not_scaled_by_dt", "const double u = dtv * xt[p];", "const double u = xt[p];"),
    ("decay_sign_flipped", "const double a = exp(dtv * A[h]);\n        const double* xt",
     "const double a = exp(-dtv * A[h]);\n        const double* xt"),
    ("initial_state_ignored", "    if (init)\n        memcpy", "    if (0)\n        memcpy"),
    ("decay_uses_previous_dt",
     "const double a = exp(dtv * A[h]);\n        const double* xt",
     "const double a = exp((t > 0 ? dt[(b * seqlen + t - 1) * nheads + h] : dtv) * A[h]);\n"
     "        const double* xt"),
]


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, source, name, old, new):
    assert source.count(old) == 1, f"mutation site for {name} not unique in ssd_oracle.c"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", str(lib),
                    str(src), "-lm"], check=True)
    failed = pins.run_all(oracle.recurrence_from(str(lib)))
    assert failed, f"no pin caught the planted mistake '{name}'"
