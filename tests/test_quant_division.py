"""Host check of the chunk path's activation quantizer division (no GPU).

The quantizer divides each value of a 16-value block by d = e4m3(s) * a_g.  Instead of 16 IEEE
divisions it takes the correctly rounded reciprocal once and corrects each product with two FMA
remainder steps (Markstein 1990).  The plain-C program below replays that sequence in IEEE fp32
(gcc, FMA from libm, no contraction) over every finite bf16 value against the divisors of eight
a_g values (two fixed, six drawn) and requires the IEEE quotient bit for bit wherever it can give
a nonzero E2M1 code; the exhaustive run over 400 a_g values found no difference either.
"""
import os
import shutil
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_reciprocal_division_matches_ieee(tmp_path):
    exe = tmp_path / "division_check"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                    os.path.join(HERE, "native", "division_check.c"), "-lm"], check=True)
    r = subprocess.run([str(exe), "8", "7"], capture_output=True, text=True, timeout=600)
    sys.stdout.write(r.stdout)
    assert r.returncode == 0, r.stdout
    assert "0 differ" in r.stdout
