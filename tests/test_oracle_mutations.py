"""The pins must catch plausible mistakes: each case plants one in a copy of the oracle's
C source (on the CPU), builds it, and runs the pin suite against it; the suite must fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

MUTATIONS = {
    # the error term predicts with the undecayed state (alpha applied after the write)
    "undecayed_prediction": ("b * (vt[i] - p[i])", "b * (vt[i] - p[i] / alpha)"),
    "error_sign": ("b * (vt[i] - p[i])", "b * (vt[i] + p[i])"),
    "dropped_beta": ("const double err = b * (vt[i] - p[i]);", "const double err = (vt[i] - p[i]);"),
    "transposed_readout": ("acc += S[(int64_t)i * dk + j] * qh[j];", "acc += S[(int64_t)j * dk + i] * qh[j];"),
    "reversed_taps": ("z += w[(int64_t)c * 4 + j]", "z += w[(int64_t)c * 4 + (3 - j)]"),
    "missing_silu": ("return z / (1.0 + exp(-z));", "return z;"),
    "eps_outside_sqrt": ("1.0 / sqrt(ss + eps)", "1.0 / (sqrt(ss) + eps)"),
    "wrong_k_head_map": ("hk = h / G;", "hk = h % J->Hk;"),
    "state_taps_reversed": ("return taps[j * (int64_t)Cc + c];", "return taps[(2 - j) * (int64_t)Cc + c];"),
    "decay_missing": ("S[e] *= alpha;", "S[e] *= 1.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(lib),
                           str(mutant), "-lm", "-lpthread"])
    env = dict(os.environ, GDN_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch '{name}':\n{r.stdout[-2000:]}"
