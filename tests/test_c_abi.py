"""The boundary from a plain C caller: tests/c_abi_consumer.c includes
include/attn.h, is compiled as strict C11 (-pedantic -Werror) and linked
against the in-tree libattn.so, then run.  It makes no GPU call."""
import os
import shutil
import subprocess

import pytest

import exact_tiled_attention_44_b200 as A

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_consumer_compiles_links_and_runs(tmp_path):
    lib = A.library_path()
    if not os.path.exists(lib):
        A.load_library()      # raises with the build hint
    exe = tmp_path / "consumer"
    cmd = ["gcc", "-std=c11", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_consumer.c"),
           "-L", os.path.dirname(lib), "-lattn", "-Wl,-rpath," + os.path.dirname(lib), "-lm",
           "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "failures 0" in run.stdout
