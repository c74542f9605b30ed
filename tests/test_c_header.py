"""The C ABI from C: tests/c_abi_check.c, a plain C99 program, compiles
against include/gqe.h with warnings as errors (-pedantic), links against
libgqe.so and runs its argument checks (no call reaches the GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "moe_gqa_query_b200")


def test_header_is_c99_and_the_library_links_from_c(tmp_path):
    gcc = shutil.which("gcc")
    if not gcc:
        pytest.skip("needs gcc")
    if not os.path.exists(os.path.join(PKG, "libgqe.so")):
        pytest.skip("the library is not built")
    exe = str(tmp_path / "c_abi_check")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", PKG, "-lgqe", "-Wl,-rpath," + PKG,
           "-Wl,--allow-shlib-undefined", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c-abi: ok" in r.stdout, r.stdout + r.stderr
