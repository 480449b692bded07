"""The per-row divisions of the fused producers (x / r of RMSNorm, h / s of
the quantisation) use Markstein's correction from a correctly rounded
reciprocal instead of a division instruction. This CPU test checks that the
correction gives the correctly rounded binary32 quotient on every FP16
numerator against 2000 divisors and on every FP16 scale against 200
numerators each (tests/csrc/recip_division_check.c states the sweeps)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _build(tmp_path, *defines):
    exe = str(tmp_path / ("recip_division_check" + "".join(defines)))
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", *defines, "-o", exe,
                           os.path.join(HERE, "csrc", "recip_division_check.c"), "-lm"])
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_markstein_quotient_is_correctly_rounded(tmp_path):
    out = subprocess.run([_build(tmp_path), "2000", "200"], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout
    assert out.stdout.strip().startswith("mismatches 0 of")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_the_sweeps_catch_a_missing_correction(tmp_path):
    """Planted on the CPU: without the FMA correction the product q0 = a * y is
    often one ulp off, and the sweeps must say so."""
    out = subprocess.run([_build(tmp_path, "-DPLANT_NO_CORRECTION"), "200", "20"], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 1
    bad = int(out.stdout.strip().splitlines()[-1].split()[1])
    assert bad > 1000
