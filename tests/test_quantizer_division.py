"""The quantizer's clip search rounds w / s to a code for every weight and every ratio.
The kernel forms that quotient from the scale's reciprocal and one exact FMA correction
instead of an IEEE division. This host check runs that arithmetic over the whole input
domain the fast path accepts (every finite fp16 scale, every finite bf16 weight with
|w| / s below 2^126) and requires the rounded quotient, which is all that reaches a code,
to equal the rounded IEEE quotient everywhere. The GPU tests then compare the kernel's
codes, scales and zeros with the oracle's bit for bit."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_reciprocal_correction_rounds_like_division(tmp_path):
    exe = tmp_path / "check"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-o", str(exe),
                           os.path.join(HERE, "quantizer_division_check.c"), "-lm"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    words = out.stdout.split()
    pairs, bad = int(words[0]), int(words[5])
    assert pairs > 2 * 10 ** 9 and bad == 0, out.stdout
