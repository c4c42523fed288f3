"""The C ABI from C++: tests/abi_check.cpp is compiled against
include/bitlinear.h with g++ and linked to libbitlinear.so.  The host checks
run here (no GPU); the GPU run adds an INT32 forward compared with a brute
force computed in the C++ program itself."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "bitlinear_b1_fwd_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def abi_binary(tmp_path_factory):
    from bitlinear_b1_fwd_b200 import build
    lib = build.build()
    exe = str(tmp_path_factory.mktemp("abi") / "abi_check")
    cmd = ["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "abi_check.cpp"), "-o", exe,
           lib, f"-Wl,-rpath,{LIBDIR}", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    subprocess.run(cmd, check=True)
    return exe


def test_host_checks_from_cpp(abi_binary):
    r = subprocess.run([abi_binary], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("OK")


@pytest.mark.gpu
def test_forward_from_cpp(abi_binary):
    r = subprocess.run([abi_binary, "--gpu"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("OK")
