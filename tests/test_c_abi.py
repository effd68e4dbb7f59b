"""The C ABI used from plain C: tests/c/abi_host_check.c is compiled with gcc against
include/fused_norm.h alone (no CUDA headers) and linked to the in-tree library, then run.
It exercises the host-only entry points (create, get_config, validate, plan, an empty
launch, status strings, version, destroy); nothing touches a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "rmsnorm_row_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_against_the_header(tmp_path):
    assert os.path.exists(os.path.join(PKG, "libfused_norm.so")), "build the library first"
    exe = tmp_path / "abi_host_check"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                         "-I", os.path.join(ROOT, "include"),
                         os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-o", str(exe),
                         "-L", PKG, "-lfused_norm", f"-Wl,-rpath,{PKG}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "0 failure(s)" in run.stdout
