"""The C ABI from plain C: tests/c/abi_check.c is compiled as C99 against
include/attn.h, linked against the in-tree libattn.so and run (no GPU
needed; it exercises only the argument checks and size formulas)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_library_links(tmp_path):
    import __graft_entry__
    __graft_entry__.build()
    libdir = os.path.join(ROOT, "scaled_dot_product_saving_b200")
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", exe,
           os.path.join(libdir, "libattn.so"), "-Wl,-rpath," + libdir]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "abi_check ok" in run.stdout
