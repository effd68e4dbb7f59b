"""The C ABI used from plain C.

tests/c/abi_host_check.c is compiled with gcc against include/fused_norm.h alone (no CUDA
headers) and linked to the in-tree library, then run: it exercises the host-only entry
points (create, get_config, validate, plan, an empty launch, status strings, version,
destroy); nothing touches a GPU. tests/c/abi_gpu_check.c runs the whole path from C on a
GPU (runtime allocations, one launch, copies back); its outputs are compared with the fp64
oracle's on the same inputs."""
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


CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build_gpu_check(tmp_path):
    exe = tmp_path / "abi_gpu_check"
    cc = subprocess.run(["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror",
                         "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA_HOME, "include"),
                         os.path.join(ROOT, "tests", "c", "abi_gpu_check.c"), "-o", str(exe),
                         "-L", PKG, "-lfused_norm", f"-Wl,-rpath,{PKG}",
                         "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart",
                         f"-Wl,-rpath,{os.path.join(CUDA_HOME, 'lib64')}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.exists(os.path.join(CUDA_HOME, "include")),
                    reason="needs gcc and the CUDA headers")
def test_c_gpu_program_builds(tmp_path):
    # the GPU-side C caller compiles cleanly against the header and the CUDA runtime API
    assert os.path.exists(os.path.join(PKG, "libfused_norm.so")), "build the library first"
    _build_gpu_check(tmp_path)


@pytest.mark.gpu
def test_c_gpu_program_matches_the_oracle(tmp_path):
    # a plain C program allocates with the CUDA runtime, launches through the C ABI and
    # copies back; its y and r equal the fp64 oracle's on the same inputs, bit for bit
    import numpy as np

    import oracle
    exe = _build_gpu_check(tmp_path)
    L, D = 37, 5120
    fin, fout = tmp_path / "in.bin", tmp_path / "out.bin"
    run = subprocess.run([str(exe), str(L), str(fin), str(fout)], capture_output=True, text=True,
                         timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    h = np.fromfile(fin, dtype=np.uint16)
    o = np.fromfile(fout, dtype=np.uint16)
    n = L * D
    x, res, gate, w = h[:n], h[n:2 * n], h[2 * n:2 * n + D], h[2 * n + D:2 * n + 2 * D]
    s, t = h[2 * n + 2 * D:3 * n + 2 * D], h[3 * n + 2 * D:4 * n + 2 * D]
    st, b0 = (L * D, 0, D), (0, 0, 0)
    ref = oracle.fused_norm(1, L, D, x=x, x_st=st, residual=res, res_st=st, gate=gate, gate_st=b0,
                            weight=w, scale=s, scale_st=st, shift=t, shift_st=st, eps=1e-6)
    assert np.array_equal(o[:n], ref["y"].reshape(-1))
    assert np.array_equal(o[n:], ref["r"].reshape(-1))
