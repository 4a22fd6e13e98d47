"""The oracle and the CUDA path share no code and neither reaches into the other.

The product (the package, its CUDA sources and the C header) must not import, include, link
or name the oracle; the oracle must not include the CUDA sources or the header, nor import the
package.  The input generator that feeds both holds none of the layer's arithmetic, and the
product path fails loudly without its CUDA library (checked in test_abi.py).
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixture_experts_ffn_13_b200")


def _files(top, exts):
    for d, _, names in os.walk(top):
        if "_build" in d:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_product_does_not_reach_the_oracle():
    pat = re.compile(r"\boracle\b|orc_|liboracle|moe_oracle")
    hits = []
    for path in list(_files(PKG, (".py", ".cu", ".cuh", ".h"))) + list(_files(os.path.join(ROOT, "include"), (".h",))):
        with open(path, encoding="utf-8") as f:
            for i, line in enumerate(f, 1):
                if pat.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{i}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_oracle_does_not_reach_the_product():
    pat = re.compile(r"mixture_experts_ffn_13_b200|moe_b200\.h|csrc|#include\s+\"")
    hits = []
    for path in _files(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        with open(path, encoding="utf-8") as f:
            for i, line in enumerate(f, 1):
                if pat.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{i}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_input_generator_imports_neither_side():
    with open(os.path.join(ROOT, "moe_synth", "__init__.py"), encoding="utf-8") as f:
        src = f.read()
    assert not re.search(r"^\s*(import|from)\s+(oracle|mixture_experts_ffn_13_b200)\b", src, re.M)
