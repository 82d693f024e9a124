"""The boundary from plain C: tests/c_client.c is compiled as C99 by gcc against
include/qwen3_attn.h alone, linked with libqwen3attn.so and run.  It checks that the
header is valid C (no C++ or CUDA types leak into it) and that a C program can call the
library: version and status strings, size helpers and host argument checks, none of which
needs a GPU.  A second probe prints the C layout of the structs passed by pointer, which
the binding's ctypes Structures must reproduce."""
import ctypes
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


LAYOUT_C = r"""
#include <stddef.h>
#include <stdio.h>
#include "qwen3_attn.h"
#define F(T, f) printf("%s.%s %zu %zu\n", #T, #f, offsetof(T, f), sizeof(((T*)0)->f))
int main(void) {
  F(qwen3_attn_variant, theta); F(qwen3_attn_variant, inv_freq);
  F(qwen3_attn_variant, attention_scaling); F(qwen3_attn_variant, window);
  F(qwen3_paged_kv, k_pages); F(qwen3_paged_kv, v_pages); F(qwen3_paged_kv, block_table);
  F(qwen3_paged_kv, num_pages); F(qwen3_paged_kv, page_size); F(qwen3_paged_kv, max_blocks);
  printf("qwen3_attn_variant %zu\nqwen3_paged_kv %zu\n", sizeof(qwen3_attn_variant), sizeof(qwen3_paged_kv));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed to build the layout probe")
def test_struct_layouts_match_the_binding(tmp_path):
    """The structs passed by pointer across the ABI have, field by field, the offsets and
    sizes the ctypes Structures of the binding assume (C compiler's layout, printed by a
    tiny program built against the header)."""
    src = tmp_path / "layout.c"
    src.write_text(LAYOUT_C)
    exe = str(tmp_path / "layout")
    res = subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", exe],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    c = {}
    for line in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.splitlines():
        key, *vals = line.split()
        c[key] = tuple(int(v) for v in vals)
    for cname, cls in (("qwen3_attn_variant", qa.Variant), ("qwen3_paged_kv", qa.PagedKV)):
        assert [f for f, _ in cls._fields_] == [k.split(".")[1] for k in c if k.startswith(cname + ".")]
        for field, ftype in cls._fields_:
            got = (getattr(cls, field).offset, ctypes.sizeof(ftype))
            assert got == c[f"{cname}.{field}"], (cname, field, got)
        assert ctypes.sizeof(cls) == c[cname][0]
