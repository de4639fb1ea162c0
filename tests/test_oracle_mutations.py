"""Each planted mistake in a copy of the oracle fails at least one of the oracle's pins.

The pins of tests/test_oracle_*.py are only worth something if a plausible error in the
oracle breaks one of them. Every case below copies `oracle/`, `synth/` and the pin files
to a temporary directory, plants one mistake in the copy (a transposed operand, a wrong
scale, a dropped factor, a wrong tie rule or exponent, a missing sign fix) and runs the
pins of the planted file there; the run must fail. The repository's own oracle is never
touched. The planted mistakes run in parallel subprocesses.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (file, text, replacement, pin file): the mistake is the first occurrence of `text`
# replaced by `replacement`.
MUTATIONS = [
    # reconstruction un-rotates with Pi instead of Pi^T
    ("oracle/quantizer.py", "(yt @ np.asarray(Pi, np.float64))", "(yt @ np.asarray(Pi, np.float64).T)",
     "tests/test_oracle_quantizer.py"),
    # QJL scale sqrt(2/pi)/d instead of sqrt(pi/2)/d (Definition 1)
    ("oracle/quantizer.py", "np.sqrt(np.pi / 2.0) / d", "np.sqrt(2.0 / np.pi) / d", "tests/test_oracle_quantizer.py"),
    # sign(S^T r) instead of sign(S r)
    ("oracle/quantizer.py", "s = r @ np.asarray(S, np.float64).T", "s = r @ np.asarray(S, np.float64)",
     "tests/test_oracle_quantizer.py"),
    # QJL reconstruction with S in place of S^T
    ("oracle/quantizer.py", "* (sgn @ S)", "* (sgn @ S.T)", "tests/test_oracle_quantizer.py"),
    # ||r|| dropped from the QJL term
    ("oracle/quantizer.py", "(np.asarray(rnorms, np.float64) * QJL_SCALE(d))",
     "(QJL_SCALE(d) + 0 * np.asarray(rnorms, np.float64))", "tests/test_oracle_quantizer.py"),
    # a value on a boundary goes to the lower cell
    ("oracle/quantizer.py", 'side="right"', 'side="left"', "tests/test_oracle_quantizer.py"),
    # boundaries off the midpoints
    ("oracle/codebook.py", "t = 0.5 * (c[:-1] + c[1:])", "t = 0.45 * (c[:-1] + c[1:])", "tests/test_oracle_codebook.py"),
    # Lemma-1 exponent (d - 2)/2 instead of (d - 3)/2
    ("oracle/codebook.py", "(d - 3) / 2.0)", "(d - 2) / 2.0)", "tests/test_oracle_codebook.py"),
    # QR without the sign fix of the Haar rotation
    ("oracle/rotation.py", "return q * s[None, :]", "return q", "tests/test_oracle_rotation.py"),
    # RHT signs applied to the rows instead of the columns
    ("oracle/rotation.py", "* eps[None, :]", "* eps[:, None]", "tests/test_oracle_rotation.py"),
    # softmax of slightly scaled scores
    ("oracle/attention.py", "m = np.max(s, axis=axis, keepdims=True)",
     "m = np.max(s, axis=axis, keepdims=True); s = s * 1.01", "tests/test_oracle_attention.py"),
]


def _run_planted(case, base):
    i, (fname, old, new, pins) = case
    work = os.path.join(base, f"m{i}")
    os.makedirs(work)
    for sub in ("oracle", "synth"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(work, sub))
    os.makedirs(os.path.join(work, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(work, "tests", "golden"))
    for f in ("conftest.py", os.path.basename(pins)):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(work, "tests", f))
    path = os.path.join(work, fname)
    with open(path) as f:
        text = f.read()
    if old not in text:
        return i, "missing"
    with open(path, "w") as f:
        f.write(text.replace(old, new, 1))
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1", OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", pins, "-q", "-x", "-p", "no:cacheprovider"], cwd=work,
                       env=env, capture_output=True, text=True, timeout=900)
    return i, r.returncode


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = str(tmp_path_factory.mktemp("planted"))
    workers = max(1, min(len(MUTATIONS), (os.cpu_count() or 2)))
    with cf.ThreadPoolExecutor(workers) as ex:
        return dict(ex.map(lambda c: _run_planted(c, base), enumerate(MUTATIONS)))


@pytest.mark.parametrize("i", range(len(MUTATIONS)), ids=[m[0].split("/")[1] + f"-{k}" for k, m in enumerate(MUTATIONS)])
def test_planted_mistake_fails_a_pin(outcomes, i):
    rc = outcomes[i]
    assert rc != "missing", f"the text to plant is no longer in {MUTATIONS[i][0]}: {MUTATIONS[i][1]!r}"
    # pytest exits 1 when a test failed (2-5 would be a collection or usage error)
    assert rc == 1, f"planted mistake {MUTATIONS[i][1]!r} -> {MUTATIONS[i][2]!r} passed every pin (rc {rc})"
