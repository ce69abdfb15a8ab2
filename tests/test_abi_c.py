"""libhadq from plain C: tests/c/abi_smoke.c is compiled with gcc against
include/hadq.h, linked to the in-tree libhadq.so and run.  The host checks
need no GPU; the GPU variant rotates and quantizes basis vectors on the
device and compares with their closed form."""

import os
import shutil
import subprocess

import pytest

from hadamard_rotation_bit_b200 import build as hbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    lib = hbuild.build()
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    exe = str(tmp_path / "abi_smoke")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "abi_smoke.c"),
           "-L", libdir, "-l:libhadq.so", f"-Wl,-rpath,{libdir}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-lm",
           "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return exe


def test_c_program_host_checks(tmp_path):
    exe = _compile(tmp_path)
    res = subprocess.run([exe, "host"], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "abi_smoke ok" in res.stdout


@pytest.mark.gpu
def test_c_program_on_the_gpu(tmp_path):
    exe = _compile(tmp_path)
    res = subprocess.run([exe, "gpu"], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "abi_smoke ok (gpu)" in res.stdout
