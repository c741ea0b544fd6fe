"""The activation quantiser's divide-free quotients equal the IEEE divides
over their whole input domain: the codes for every BF16 value against every
scale a BF16 group maximum produces (scales >= 2^-100), and the scale
amax/448 for every BF16 amax.  The comparison runs on the
host in IEEE binary32 (tests/exact_quotient_check.c); the GPU parity tests
then compare the kernel's codes with the oracle's IEEE divide."""
import os
import re
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_divide_free_quotient_exhaustive(tmp_path):
    exe = tmp_path / "exact_quotient_check"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-o", str(exe),
                    os.path.join(HERE, "exact_quotient_check.c"), "-lm"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=600).stdout
    m = re.search(r"pairs=(\d+) code_mismatch=(\d+) float_mismatch=(\d+) scales=(\d+) scale_mismatch=(\d+)", out)
    assert m, out
    pairs, code_bad, float_bad, scales, scale_bad = (int(g) for g in m.groups())
    # every positive finite BF16 amax with s >= 2^-100 and every BF16 |x| <= amax, both signs
    assert pairs > 1_000_000_000
    assert code_bad == 0, out
    # the floats themselves differ only for a small set of subnormal-range quotients
    assert float_bad < pairs // 100
    # the group scale RN(amax/448): every finite non-negative BF16 amax, bit for bit
    assert scales == 0x7F80 and scale_bad == 0, out
