"""The oracle pins catch plausible mistakes.

Each case copies the oracle's C source, plants one mistake (a flipped sign, a
dropped normalisation, a wrong divisor, a wrong index, a missing stage, an
off-by-one partial sum), compiles it to a temporary library and reruns the pin
suite against it in a subprocess: the suite must fail.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as ob

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    ("butterfly sign", "v[j + h] = a - b;", "v[j + h] = b - a;"),
    ("normalisation dropped", "out[t * (int64_t)K + j] = row[j] * c;", "out[t * (int64_t)K + j] = row[j];"),
    ("quantiser divisor", "float scale = amax / 7.0f;", "float scale = amax / 8.0f;"),
    ("group index", "if (a > s[j / G]) s[j / G] = a;", "if (a > s[j % (K / G)]) s[j % (K / G)] = a;"),
    ("last stage missing", "for (int h = 1; h < n; h *= 2) {", "for (int h = 1; h < n / 2; h *= 2) {"),
    ("partial sum off by one", "P[((int64_t)g * R + i) * N + c] = (int32_t)acc;",
     "P[((int64_t)g * R + i) * N + c] = (int32_t)(acc + 1);"),
    ("smoothing skipped", "z[j] = Xp[t * (int64_t)K + j] / d;", "z[j] = Xp[t * (int64_t)K + j];"),
    ("packing swapped", "out[i] = (uint8_t)(((uint8_t)q[2 * i] & 0x0Fu) | (((uint8_t)q[2 * i + 1] & 0x0Fu) << 4));",
     "out[i] = (uint8_t)(((uint8_t)q[2 * i + 1] & 0x0Fu) | (((uint8_t)q[2 * i] & 0x0Fu) << 4));"),
]


PIN_SUITES = ["test_oracle_pins.py", "test_oracle_golden.py"]


@pytest.mark.parametrize("suite", PIN_SUITES)
@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_fail_on_planted_mistake(tmp_path, name, old, new, suite):
    """Both the pin suite and the hand-worked example, each on its own, catch every mistake."""
    src = open(ob.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found for {name}"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", *ob.CFLAGS, str(mut), "-o", str(lib), "-lm"])
    env = dict(os.environ, RRS_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", suite)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation '{name}':\n{r.stdout[-2000:]}"
