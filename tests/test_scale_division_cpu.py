"""The append kernels form the scale amax/448 as a product with RN(1/448)
corrected by one FMA residual step (Markstein's correction) instead of a
division.  This pins that it equals IEEE division for every float from 2^-120
up (the kernels divide below that), exhaustively, on the host's IEEE FMA."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _has_fma() -> bool:
    try:
        return " fma " in open("/proc/cpuinfo").read().replace("\n", " ")
    except OSError:
        return False


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_corrected_reciprocal_equals_division_exhaustively():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "div448")
        flags = ["-O2", "-ffp-contract=off", "-fopenmp"] + (["-mfma"] if _has_fma() else [])
        subprocess.check_call(["gcc", *flags, os.path.join(HERE, "div448_check.c"), "-o", exe, "-lm"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=600)
        checked, bad = (int(x) for x in out.stdout.split())
        assert checked == 0x7F800000 - 0x03800000
        assert bad == 0 and out.returncode == 0
