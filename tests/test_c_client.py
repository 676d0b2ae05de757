"""The boundary is a plain C ABI: a C program that includes only
include/gdr2.h and links libgdr2.so builds with gcc and passes its host-side
checks (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import linear_attention_recurrence_gdr2_b200 as gdr2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_client_builds_and_passes(tmp_path):
    lib_dir = os.path.dirname(gdr2.LIB_PATH)
    exe = tmp_path / "abi_host"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", lib_dir, "-lgdr2",
           f"-Wl,-rpath,{lib_dir}", "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == "ok"
