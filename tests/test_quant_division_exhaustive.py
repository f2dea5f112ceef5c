"""The quantizer divides w by the block maximum a with Markstein's FMA
correction of a table reciprocal (see csrc/division_check.c for the method
and its reference).  This compiles and runs an exhaustive host check: for every
pair of bf16 values with 2^-64 <= a <= 2^64 and |w| <= a (both signs), the fast
quotient and the IEEE quotient give the same NF4 code.  The thresholds come
from the oracle's level table."""
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import nf4

HERE = os.path.dirname(os.path.abspath(__file__))


def _thresholds():
    L = nf4.nf4_levels().astype(np.float64)
    mid = (L[1:] + L[:-1]) / 2
    T = mid.astype(np.float32)
    T = np.where(T.astype(np.float64) > mid, np.nextafter(T, np.float32(-np.inf)), T)
    return [float(t).hex() for t in T]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_fast_division_gives_ieee_codes_for_every_bf16_pair():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "division_check")
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", os.path.join(HERE, "csrc", "division_check.c"),
                        "-o", exe, "-lm"], check=True)
        res = subprocess.run([exe] + _thresholds(), capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    fields = res.stdout.split()
    assert int(fields[1]) > 5e8                       # all pairs of the fast range were visited
    assert fields[-1] == "0"                          # no code mismatch
