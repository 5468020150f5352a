"""Host-side helpers of bench.py that decide what a bench line reports (no GPU)."""
from __future__ import annotations

import os
import shutil

import bench

SRC = """// header comment
#include "x.cuh"
__device__ int f(int a) {  // trailing comment
  asm("mov.u32 %0, %1; // not a comment inside the string" : "=r"(a) : "r"(a));

  return a + 1;
}
"""


def test_code_lines_drops_comments_and_blank_lines_only():
    code = bench.code_lines(SRC)
    assert "header comment" not in code and "trailing comment" not in code
    assert "// not a comment inside the string" in code  # a string keeps its // text
    assert "return a + 1;" in code and "" not in code.split("\n")


def _hash_of(tmp_path, files):
    d = tmp_path / "csrc"
    if d.exists():
        shutil.rmtree(d)
    d.mkdir()
    for name, text in files.items():
        (d / name).write_text(text)
    old = bench.DOMINANT_KERNEL_SRC
    bench.DOMINANT_KERNEL_SRC = str(d)
    try:
        return bench.kernel_source_hash()
    finally:
        bench.DOMINANT_KERNEL_SRC = old


def test_source_hash_ignores_comment_edits_but_not_code_edits(tmp_path):
    base = _hash_of(tmp_path, {"k.cu": SRC})
    assert _hash_of(tmp_path, {"k.cu": SRC.replace("header comment", "reworded note")}) == base
    assert _hash_of(tmp_path, {"k.cu": SRC + "\n// one more note\n"}) == base
    assert _hash_of(tmp_path, {"k.cu": SRC.replace("a + 1", "a + 2")}) != base
    assert _hash_of(tmp_path, {"k.cu": SRC, "other.cuh": "int g;\n"}) != base


def test_recorded_traffic_matches_the_current_sources():
    # the committed ncu traffic is only reported while it was taken on this code
    rec = bench.recorded_traffic(bench.HEADLINE.name)
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    assert os.path.exists(path)
    assert rec is None or rec > 0
