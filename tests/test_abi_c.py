"""The C ABI from plain C (no Python, no torch types): gcc compiles a small program against
include/svdq.h, links libsvdq.so and calls the host-side entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from bit_w4a4_quantized_group_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_host_calls_from_plain_c(tmp_path):
    lib = BUILD.build()
    exe = tmp_path / "abi_smoke"
    cmd = ["gcc", "-std=c99", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_smoke.c"), "-o", str(exe),
           "-L", os.path.dirname(lib), "-lsvdq", "-Wl,-rpath," + os.path.dirname(lib), "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.stdout, r.stderr)
