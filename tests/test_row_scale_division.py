"""The FP8 row quantizer divides by the row scale through the row's reciprocal and one
exact FMA correction step instead of an IEEE division per element. This host check runs
that arithmetic over the quantizer's whole input domain (every finite bf16 row maximum,
every bf16 value under it) and requires the E4M3-relevant result to equal the IEEE
quotient everywhere. The GPU tests then compare the kernel's codes with the oracle's."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_reciprocal_correction_equals_division(tmp_path):
    exe = tmp_path / "check"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-o", str(exe),
                           os.path.join(HERE, "row_scale_division_check.c"), "-lm"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    pairs, diffs = out.stdout.split()[0], out.stdout.split()[2]
    assert int(pairs) > 10 ** 9 and int(diffs) == 0, out.stdout
