"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of ``oracle/gspn_oracle.cpp``
(on the CPU; nothing here touches a GPU), builds the copy, and runs the pin
suites (``tests/test_oracle_pins.py``, ``tests/test_oracle_backward_pins.py``
and ``tests/test_oracle_band_pins.py``) against it in a subprocess.  The pins must
fail for every mistake.  A case whose original text is no longer in the
source fails too, so the list follows the oracle as it changes.
"""
import os
import pathlib
import shutil
import subprocess
import sys

import pytest

ROOT = pathlib.Path(__file__).resolve().parent.parent

# (name, original text, planted mistake)
MUTATIONS = [
    ("reverse scans restart from the wrong end",
     "return (d == 0 || d == 2) ? i : L() - 1 - i;", "return i;"),
    ("missing neighbour kept in the normaliser",
     "if (kn < 0 || kn >= K) continue;          // missing neighbour: dropped",
     "if (false) continue;"),
    ("first line without lambda",
     "cur[k] = drive;", "cur[k] = x[p];"),
    ("in-place update reads the new line",
     "acc += w[slot] * prev[kn];", "acc += w[slot] * (kn < k ? cur[kn] : prev[kn]);"),
    ("sigmoid with the wrong sign",
     "return 1.0 / (1.0 + std::exp(-z));", "return 1.0 / (1.0 + std::exp(z));"),
    ("slots mirrored",
     "int64_t kn = k + slot - 1;", "int64_t kn = k - slot + 1;"),
    ("left-to-right scan runs right to left",
     "case 2: return k * W + i;", "case 2: return k * W + (W - 1 - i);"),
    ("u of the wrong direction",
     "const double* ud = u[d] + q * HW;", "const double* ud = u[(d + 1) % 4] + q * HW;"),
    # backward
    ("sigmoid derivative factor dropped",
     "dz3[slot * HW + p] = w[slot] * (1.0 - sg) * (dw[slot] - dw_dot_w);",
     "dz3[slot * HW + p] = w[slot] * (dw[slot] - dw_dot_w);"),
    ("adjoint carried to the wrong neighbour",
     "carry[kn] += w[slot] * a[k];", "carry[k] += w[slot] * a[k];"),
    ("gate gradient uses the current line",
     "dw[slot] = a[k] * h[dir.pixel(i - 1, kn)];", "dw[slot] = a[k] * h[dir.pixel(i, kn)];"),
    # wider neighbourhoods
    ("band: neighbours outside the line kept in the normaliser",
     "sig[s] = (src >= 0 && src < K) ? logistic(zb[s * HW + p]) : 0.0;",
     "sig[s] = logistic(zb[s * HW + p]);"),
    ("band: offsets mirrored",
     "const int64_t src = k + (s - r);", "const int64_t src = k - (s - r);"),
    ("band: in-place update reads the new line",
     "if (src >= 0 && src < K) mix += (sig[s] / norm) * before[src];",
     "if (src >= 0 && src < K) mix += (sig[s] / norm) * (src < k ? now[src] : before[src]);"),
    ("band: last offset dropped",
     "const int64_t nslot = 2 * r + 1;\n    std::vector<double> before",
     "const int64_t nslot = 2 * r;\n    std::vector<double> before"),
]


def _run_pins_on_copy(tmp_path, src):
    shutil.copytree(ROOT / "oracle", tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("_build", "__pycache__"))
    shutil.copytree(ROOT / "tests", tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))
    shutil.copy(ROOT / "pytest.ini", tmp_path / "pytest.ini")
    (tmp_path / "oracle" / "gspn_oracle.cpp").write_text(src)
    env = dict(os.environ, PYTHONPATH=str(tmp_path))
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           "tests/test_oracle_pins.py", "tests/test_oracle_backward_pins.py",
                           "tests/test_oracle_band_pins.py"],
                          cwd=tmp_path, env=env, capture_output=True, text=True, timeout=600)


def test_unmodified_copy_passes(tmp_path):
    """Control: the same harness on an unmodified copy passes, so the failures
    below come from the planted mistakes."""
    src = (ROOT / "oracle" / "gspn_oracle.cpp").read_text()
    r = _run_pins_on_copy(tmp_path, src)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name,orig,bad", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, orig, bad, tmp_path):
    src = (ROOT / "oracle" / "gspn_oracle.cpp").read_text()
    assert orig in src, f"mutation '{name}' no longer matches the oracle source"
    r = _run_pins_on_copy(tmp_path, src.replace(orig, bad))
    assert r.returncode != 0, f"pins pass with mistake '{name}':\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
