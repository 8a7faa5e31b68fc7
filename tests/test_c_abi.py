"""The boundary as a C client sees it: tests/c_abi_check.c, which includes
only include/isa.h, compiles as strict C99 (-Wall -Wextra -pedantic
-Werror), links against the built libisa.so with no C++ or CUDA flags and
runs its host-side checks (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)


@pytest.fixture(scope="module")
def libdir():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    return os.path.join(ROOT, "block_sparse_attention_coarse_b200")


def test_c_client_builds_links_and_runs(libdir, tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    assert cc, "a C compiler is needed"
    exe = str(tmp_path / "c_abi_check")
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(TESTS, "c_abi_check.c"), "-o", exe, "-L", libdir, "-l:libisa.so", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
