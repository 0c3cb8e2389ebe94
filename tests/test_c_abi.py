"""The boundary from C: ``tests/c/abi_check.c`` is compiled against
``include/moe.h`` as strict C99 and as C++17 (warnings are errors), linked
with the built library and run.  It exercises only host-side behaviour (plan
checks, status names, argument checks that fail before any launch), so it
needs no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
PKG = os.path.join(ROOT, "moe_expert_ffn_permute_b200")
LIB = os.path.join(PKG, "libmoe_b200.so")


@pytest.mark.parametrize("compiler,flags", [
    ("gcc", ["-std=c99", "-pedantic"]),
    ("g++", ["-x", "c++", "-std=c++17"]),
], ids=["c99", "c++17"])
def test_c_program_against_the_header(tmp_path, compiler, flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    if not os.path.exists(LIB):
        from moe_expert_ffn_permute_b200 import build
        build.build()
    exe = str(tmp_path / "abi_check")
    cmd = [compiler, *flags, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", PKG, "-lmoe_b200",
           f"-Wl,-rpath,{PKG}", "-lm", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("abi ok"), r.stdout + r.stderr
