"""The encoder computes fl(fl(x - z) / s) with Markstein's correction step
instead of a division.  This checks the step exhaustively on the host (every
11-bit divisor significand against every binary32 dividend significand) with
the same operation sequence in C, plus a control run without the correction
that must fail."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    exe = str(tmp_path_factory.mktemp("quot") / "quotient_check")
    subprocess.run(["gcc", "-O2", "-march=native", "-ffp-contract=off", "-fopenmp",
                    os.path.join(HERE, "exhaustive", "quotient_check.c"), "-o", exe, "-lm"],
                   check=True)
    return exe


def test_correction_step_is_correctly_rounded(checker):
    out = subprocess.run([checker], capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout
    assert out.stdout.startswith("mismatches 0 of 8589934592")


def test_control_without_correction_fails(checker):
    out = subprocess.run([checker, "skip-correction"], capture_output=True, text=True, timeout=900)
    assert out.returncode == 1
    assert not out.stdout.startswith("mismatches 0 ")
