"""The quantizers' division (csrc/quant_div.h: a reciprocal and one
correction step) equals IEEE fp32 division bit for bit on the inputs the
pre-pass gives it: every fp16 absmax / colmax, divisors with an all-ones
significand, powers of two and random fp32 divisors, V_r in {448, 9}
(tests/c/div_check.cpp, compiled as host code from the same header)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_division_equals_ieee_bit_for_bit(tmp_path):
    exe = str(tmp_path / "div_check")
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "quantized_attention_08_b200", "csrc"),
           os.path.join(ROOT, "tests", "c", "div_check.cpp"), "-o", exe, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout
    assert run.stdout.startswith("ok "), run.stdout
    assert int(run.stdout.split()[1]) > 10 ** 8
