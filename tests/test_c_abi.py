"""The C ABI from plain C: include/sage.h compiles as C99 with warnings as
errors, a C program links against libsage.so and its host-side checks
answer without a GPU (tests/c/abi_from_c.c makes only calls the checks
reject)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_checks(tmp_path):
    from quantized_attention_08_b200 import build
    build.build()
    pkg = os.path.join(ROOT, "quantized_attention_08_b200")
    exe = str(tmp_path / "abi_from_c")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-o", exe, "-L", pkg, "-lsage",
           f"-Wl,-rpath,{pkg}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("ok")
