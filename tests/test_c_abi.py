"""The C ABI from plain C: include/qlora.h compiles as C11 and as C++17, a
C program links against libqlora.so and its host-only calls behave (no GPU
needed, no torch involved)."""
import os
import shutil
import subprocess

import pytest

from qlora_bit_frozen_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "abi_check.c")
LIBDIR = os.path.join(ROOT, "qlora_bit_frozen_b200")


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-std=c11", "-x", "c"]),
                                            ("g++", ["-std=c++17", "-x", "c++"])])
def test_header_and_library_from_c(tmp_path, compiler, flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    build.build()
    exe = str(tmp_path / "abi_check")
    cmd = [compiler, "-Wall", "-Werror", *flags, "-I", os.path.join(ROOT, "include"), SRC, "-x", "none",
           "-L", LIBDIR, "-lqlora", "-Wl,-rpath," + LIBDIR, "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
