"""The C ABI from plain C: tests/c_abi_example.c compiles as C99 against
include/sv.h with warnings as errors, links libsv.so, and runs (it uses only
calls that do no CUDA work, so no GPU is needed)."""
import os
import shutil
import subprocess

import pytest

import speculative_decoding_verification_93_b200 as sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_caller(tmp_path):
    lib = sv.library_path()
    sv.lib()   # raises if the library is missing
    exe = str(tmp_path / "c_abi_example")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_example.c"), lib,
                    "-Wl,-rpath," + os.path.dirname(lib), "-o", exe], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "c abi ok"
