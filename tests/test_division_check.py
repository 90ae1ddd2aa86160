"""The quantize kernel divides without a division instruction (a correctly
rounded reciprocal, a product and Markstein's FMA correction).  This checks on
the host, in C with IEEE float operations and the C library's fmaf, that the
three steps give the IEEE quotient w / a wherever it can decide a code, on a
bounded sample of (w, a) pairs spanning the kernel's fast range of a
(2^-98 <= a < 2^120); the GPU parity tests check the codes themselves bit for
bit against the oracle."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_markstein_corrected_quotient_is_ieee(tmp_path):
    exe = str(tmp_path / "division_check")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "native", "division_check.c"), "-lm"], check=True)
    # 2000 scales x 20000 values: 4 x 10^7 pairs, a few seconds
    out = subprocess.run([exe, "2000", "20000", "7"], check=True, capture_output=True, text=True)
    pairs, bad = (int(v) for v in out.stdout.split())
    assert pairs == 2000 * 20004
    assert bad == 0, f"{bad} of {pairs} pairs differ from the IEEE quotient"
