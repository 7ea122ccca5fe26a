"""The C ABI from plain C (CPU only): tests/c/abi_host.c is compiled with gcc against
include/moe.h, linked to libmoe.so and run; it checks the host-side entry points
(version, status text, configuration checks, workspace and window sizes, the EPLB plan)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "dispatch_combine_grouped_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_against_the_abi(tmp_path):
    exe = tmp_path / "abi_host"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-o", str(exe), "-L", PKG, "-l:libmoe.so",
                    f"-Wl,-rpath,{PKG}"], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
