"""The C ABI from C: tests/c/abi_smoke.c is compiled as C99 against
include/convrot.h with gcc (-Wall -Werror), linked to the in-tree
libconvrot.so and run.  No GPU is needed: every call it makes is answered by
the host-side argument validation."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "w8a8_int8_quantized_rmsnorm_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_caller_compiles_links_and_validates(tmp_path):
    from w8a8_int8_quantized_rmsnorm_b200 import build
    build.build()
    exe = str(tmp_path / "abi_smoke")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_smoke.c"), "-L", PKG, "-lconvrot",
           f"-Wl,-rpath,{PKG}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi smoke: ok" in r.stdout
