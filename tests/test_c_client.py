"""The boundary from plain C: tests/c_client.c is compiled as C99 by gcc against
include/qwen3_attn.h alone, linked with libqwen3attn.so and run.  It checks that the
header is valid C (no C++ or CUDA types leak into it) and that a C program can call the
library: version and status strings, size helpers and host argument checks, none of which
needs a GPU."""
import os
import shutil
import subprocess

import pytest

import qwen3_qk_norm_rope_b200 as qa

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed to build the C client")
def test_plain_c_client(tmp_path):
    lib = qa.lib()._name  # loads (and thereby checks) the in-tree library
    exe = str(tmp_path / "c_client")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(HERE, "c_client.c"), "-o", exe, lib, "-Wl,-rpath," + os.path.dirname(lib)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
