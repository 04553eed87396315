"""The pre-pass kernels' paired division (csrc/quant_pair.cuh: div2_rn and
codes4) against IEEE fp32 division on the device, bit for bit, over every
fp16 input of every fp16-derived divisor (tests/c/div_check_gpu.cu); the
scalar definition it follows is checked on the host by test_quant_div.py."""
import os
import subprocess

import pytest

from quantized_attention_08_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "quantized_attention_08_b200", "csrc")


def test_paired_division_exhaustive(tmp_path):
    exe = str(tmp_path / "div_check_gpu")
    cmd = [build._nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-I", CSRC, "-o", exe, os.path.join(HERE, "c", "div_check_gpu.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    res = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and res.stdout.startswith("ok"), res.stdout[-2000:]
