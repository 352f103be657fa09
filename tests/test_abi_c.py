"""The boundary from plain C: tests/abi_c/check_abi.c is compiled with gcc as
C11 against include/moe_verify.h, linked to the library and run (no GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_caller_builds_links_and_passes(tmp_path):
    from moe_decoder_speculative_b200 import build
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "check_abi")
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "abi_c", "check_abi.c"), "-o", exe, "-L", libdir,
                           "-lmoe_verify", f"-Wl,-rpath,{libdir}"])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "C ABI checks passed" in r.stdout
