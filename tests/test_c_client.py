"""The C ABI from C: tests/c_abi_client.c includes include/pa.h as strict
C99 (-pedantic -Werror), links libpa.so and drives the host allocator
through a fork, its copy-on-write and the prefix grouping (CPU only)."""

import os
import shutil
import subprocess
import tempfile

import pytest

import paged_kv_cache_351_b200  # noqa: F401  (the library is built and loads)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "paged_kv_cache_351_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_client():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "client")
        cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                             "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_client.c"),
                             "-L", LIBDIR, "-lpa", f"-Wl,-rpath,{LIBDIR}", "-o", exe],
                            capture_output=True, text=True)
        assert cc.returncode == 0, cc.stderr
        run = subprocess.run([exe], capture_output=True, text=True, timeout=60,
                             env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
        assert run.returncode == 0, (run.returncode, run.stderr)
    # CoW pair (shared block 1 -> fresh block 2); the child's table; block 0
    # held by both; 8 - 3 blocks in use; all free again; the status text
    lines = run.stdout.splitlines()
    assert lines[0].split() == ["1", "2", "0", "2", "2", "5"]
    # prefix groups: one group of both sequences sharing block 0
    assert lines[1].split() == ["1", "0", "2", "1"]
    assert lines[2] == "8 out of free blocks"
