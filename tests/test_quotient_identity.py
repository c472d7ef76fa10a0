"""The quantization kernels divide x by the row scale s with one reciprocal
per row and two FMA roundings per element (Markstein's correction) instead
of a full division; the codes are only bit-exact if that quotient is the
correctly rounded x / s.  This checks the identity on the host, in C (IEEE
fp32 with a fused multiply-add, no contraction), for every bf16 significand
of x against every fp32 significand of s."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    exe = tmp_path_factory.mktemp("quotient") / "quotient_identity"
    flags = ["-O2", "-ffp-contract=off"]
    try:   # the hardware FMA when the CPU has one (glibc's software fmaf is also exact, only slower)
        if " fma " in open("/proc/cpuinfo").read().replace("\n", " "):
            flags.append("-mfma")
    except OSError:
        pass
    subprocess.run(["gcc", *flags, "-o", str(exe),
                    os.path.join(HERE, "quotient_identity.c"), "-lm"], check=True)
    return str(exe)


@pytest.mark.parametrize("ea,eb,step", [(0, 0, 1), (5, -9, 7), (-7, 3, 7)])
def test_fma_corrected_quotient_is_correctly_rounded(checker, ea, eb, step):
    """Every divisor significand at one exponent pair; a seventh of them at
    two others (the steps scale exactly with the exponents)."""
    r = subprocess.run([checker, str(ea), str(eb), str(step)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout
    assert "mismatches=0" in r.stdout


def test_uncorrected_product_is_caught(checker):
    """Without the correction step (q0 = RN(x RN(1/s)) alone) the check finds
    mismatches, so it can tell a wrong quotient from a right one."""
    r = subprocess.run([checker, "0", "0", "64", "plain"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 1 and "mismatches=0" not in r.stdout
