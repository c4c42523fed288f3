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


def test_header_is_plain_c99(tmp_path):
    """The header compiles as strict C99 (-Wall -Wextra -pedantic -Werror) and a
    C program links against the library and calls it."""
    from bitlinear_b1_fwd_b200 import build
    lib = build.build()
    src = tmp_path / "c_client.c"
    src.write_text('#include "bitlinear.h"\n'
                   "int main(void) {\n"
                   "  if (bitlinear_packed_row_bytes(3200, BL_PACK_I2) != 800) return 1;\n"
                   "  if (bitlinear_forward(0, BL_PACK_I2, 0, 4, 4, 0, BL_BF16, 0, 1, 0, BL_BF16, 0, 0, 0)\n"
                   "      != BL_ERR_INVALID_VALUE) return 2;\n"
                   "  return bitlinear_version() >= 100 ? 0 : 3;\n"
                   "}\n")
    exe = str(tmp_path / "c_client")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", exe, lib, f"-Wl,-rpath,{LIBDIR}"], check=True)
    assert subprocess.run([exe], timeout=60).returncode == 0
