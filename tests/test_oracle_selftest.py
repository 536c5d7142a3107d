"""The oracle's C self-test: hand-derived values checked by a C program
built with the oracle's own flags (one translation unit with it)."""

import os
import subprocess
import tempfile

from oracle import build as obuild


def test_oracle_c_selftest_passes():
    with tempfile.TemporaryDirectory() as d:
        exe = obuild.compile_selftest(os.path.join(d, "oracle_selftest"))
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "all checks hold" in r.stdout
