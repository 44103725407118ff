"""The boundary from plain C: tests/c/abi_check.c includes include/hxq.h as
C99, links libhxq.so with the C compiler and checks the argument errors of
every entry point, without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "vq_compressed_linear_b200")


def test_c_program_links_and_gets_argument_errors(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if not cc:
        pytest.skip("no C compiler")
    if not os.path.exists(os.path.join(LIBDIR, "libhxq.so")):
        pytest.fail("libhxq.so is not built")
    exe = tmp_path / "abi_check"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", str(exe),
                    "-L", LIBDIR, "-l:libhxq.so", "-Wl,-rpath," + LIBDIR], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
