"""The boundary is a plain C ABI: a C99 program compiled with gcc against include/lhcal.h (no
CUDA, torch or C++ headers) links liblhcal.so and runs its GPU-free checks (tests/c/abi_check.c);
the same program built as C++17 with g++ does too."""
import os
import shutil
import subprocess

import pytest

from scale_calibration_lh_b200 import build as B


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_client_compiles_links_and_validates(tmp_path, root_dir):
    lib = B.build()
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root_dir, "include"),
           os.path.join(root_dir, "tests", "c", "abi_check.c"), "-o", str(exe), lib,
           f"-Wl,-rpath,{os.path.dirname(lib)}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi ok" in r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_cpp_client_compiles_links_and_validates(tmp_path, root_dir):
    """The same client built as C++17: the header's declarations carry C linkage for C++ callers."""
    lib = B.build()
    exe = tmp_path / "abi_check_cpp"
    cmd = ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root_dir, "include"),
           "-x", "c++", os.path.join(root_dir, "tests", "c", "abi_check.c"), "-x", "none", lib,
           f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-4000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi ok" in r.stdout
