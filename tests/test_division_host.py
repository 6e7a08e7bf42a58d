"""Exhaustive host check of the kernels' fast division (reciprocal plus one
residual correction) against IEEE single-precision division: Int8 and E4M3
second-level constants over every fp32 significand of c1, and the quantiser's
bf16 quotients (also against exact integer division).  The checker is the C
program in host_checks/; it needs gcc and takes about half a minute."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    exe = str(tmp_path_factory.mktemp("division") / "division_check")
    subprocess.run([gcc, "-O2", "-ffp-contract=off", "-o", exe, os.path.join(HERE, "host_checks", "division_check.c"),
                    "-lm"], check=True)
    return exe


@pytest.mark.parametrize("mode", ["bf16", "int8", "e4m3"])
def test_fast_division_is_correctly_rounded(checker, mode):
    r = subprocess.run([checker, mode], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("bad 0"), r.stdout
