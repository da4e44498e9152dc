"""Host logic of bench.py that needs no GPU: the kernel-code digest that keeps
recorded ncu traffic attached to the kernels it was measured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_keeps_literals():
    src = 'int a = 1; // one\n/* block\n comment */ const char* s = "x // y /* z */";\n'
    assert bench._code_only(src) == 'int a = 1; const char* s = "x // y /* z */";'


def test_code_only_collapses_blank_space_only():
    assert bench._code_only("a  +\n\n b") == bench._code_only("a + b")
    assert bench._code_only("a+b") != bench._code_only("a + b")


def _digest_of(tmp_path, files):
    csrc = tmp_path / "int4_weight_only_gptq_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in files.items():
        (csrc / name).write_text(text)
    old = bench.ROOT
    bench.ROOT = str(tmp_path)
    try:
        return bench.kernel_source_digest()
    finally:
        bench.ROOT = old


def test_digest_ignores_comment_edits_and_sees_code_edits(tmp_path):
    base = {"k.cu": "__global__ void k(int* p) { p[0] = 1; }  // store\n", "h.cuh": "#pragma once\n"}
    commented = {"k.cu": "// a kernel\n__global__ void k(int* p) { p[0] = 1; }\n",
                 "h.cuh": "#pragma once  /* header */\n"}
    changed = {"k.cu": "__global__ void k(int* p) { p[0] = 2; }\n", "h.cuh": "#pragma once\n"}
    d0 = _digest_of(tmp_path / "a", base)
    assert _digest_of(tmp_path / "b", commented) == d0
    assert _digest_of(tmp_path / "c", changed) != d0

