"""The oracle's pins catch plausible mistakes: each case plants one mistake in a copy of the
oracle's C source on the CPU, rebuilds it in a temporary directory and runs the pins that guard
that part; every planted copy must fail them.  (The committed oracle passes the same pins.)"""
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hq_oracle.c")

MUTATIONS = [
    # name, text in the oracle, planted replacement, pins expected to fail
    ("e8_coset_A_argmin", "int j = argmax_abs(e, 8);", "int j = argmin_abs(e, 8);", "tests/test_oracle_lattice_search.py"),
    ("e8_coset_B_argmax", "int m = argmin_abs(e, 8);", "int m = argmax_abs(e, 8);", "tests/test_oracle_lattice_search.py"),
    ("e8_fix_direction", "pA[j] += 2 * toward(e[j]);", "pA[j] -= 2 * toward(e[j]);", "tests/test_oracle_lattice_search.py"),
    ("e8_dropped_distance_term", "for (int i = 0; i < d; ++i) {\n        float t = z[i] - (float)p[i];",
     "for (int i = 1; i < d; ++i) {\n        float t = z[i] - (float)p[i];", "tests/test_oracle_lattice_search.py"),
    ("d4_argmin", "int j = argmax_abs(e, 4);", "int j = argmin_abs(e, 4);", "tests/test_oracle_lattice_search.py"),
    ("a2_metric_weight", "return dP * dP + 3.0f * (dQ * dQ);", "return dP * dP + 1.0f * (dQ * dQ);",
     "tests/test_oracle_lattice_search.py"),
    ("rms_sequential_sum", "for (int h = 1; h < n; h *= 2)\n        for (int i = 0; i < n; i += 2 * h) q[i] = q[i] + q[i + h];",
     "for (int i = 1; i < n; ++i) q[0] = q[0] + q[i];", "tests/test_oracle_primitives.py"),
    ("dither_half_order", "int j = 4 * (g & 1) + i;", "int j = 4 * (1 - (g & 1)) + i;", "tests/test_oracle_dither.py"),
]


@pytest.mark.parametrize("name,old,new,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_the_pins(name, old, new, pins):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"the oracle no longer contains the text planted by {name}"
    with tempfile.TemporaryDirectory(prefix="planted_") as d:
        shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
        shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"),
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_planted_mistakes.py"))
        shutil.copytree(os.path.join(ROOT, "post_quantization_tile_b200"), os.path.join(d, "post_quantization_tile_b200"),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
        with open(os.path.join(d, "oracle", "hq_oracle.c"), "w") as f:
            f.write(src.replace(old, new, 1))
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider", pins],
                           cwd=d, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed {pins}:\n{r.stdout[-2000:]}"
