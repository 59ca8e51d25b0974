"""The header is plain C: a C99 program built with gcc against include/awq.h
and linked to the library runs the host-side checks of the entry points
(no GPU needed; no call in it reaches CUDA)."""
import os
import shutil
import subprocess

import pytest

import weight_only_int4_gemv_b200 as awq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def library():
    if not os.path.exists(awq.LIB_PATH):
        from weight_only_int4_gemv_b200 import build
        build.build()
    return awq.LIB_PATH


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c99_caller_builds_and_passes(library, tmp_path):
    exe = str(tmp_path / "abi_check")
    lib_dir = os.path.dirname(library)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", exe, library, f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi_check: ok" in r.stdout
