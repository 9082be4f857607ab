"""Structural rules of the repository, checked on the sources (CPU only).

* The product package (the binding, the CUDA sources, the build script, the
  tensor-parallel layers) neither imports, loads nor names the oracle: the
  oracle is test infrastructure and the product path has no CPU fallback.
* The oracle uses nothing from the product package: the two share no code.
* The seeded input generators hold none of the method's arithmetic (no
  quantisation, scales or E4M3 codes): they serve both sides.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fp8_quantized_gemm_ptpc_b200")


def sources(folder, exts):
    for base, dirs, files in os.walk(folder):
        dirs[:] = [d for d in dirs if not d.startswith(("_build", "_lib", "__pycache__"))]
        for f in files:
            if f.endswith(exts):
                yield os.path.join(base, f)


def test_product_package_does_not_use_the_oracle():
    hits = []
    for path in sources(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        for i, line in enumerate(open(path, encoding="utf-8"), 1):
            if re.search(r"\boracle\b", line, re.IGNORECASE):
                hits.append(f"{os.path.relpath(path, ROOT)}:{i}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_oracle_does_not_use_the_product_package():
    hits = []
    for path in sources(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        text = open(path, encoding="utf-8").read()
        for pat in (r"fp8_quantized_gemm_ptpc_b200", r"\bcsrc\b", r"libptpc", r"#include\s+\"(?!math|stdint|string)"):
            for m in re.finditer(pat, text):
                hits.append(f"{os.path.relpath(path, ROOT)}: {m.group(0)}")
    assert not hits, "\n".join(hits)


def test_input_generators_hold_no_method_arithmetic():
    import ast
    tree = ast.parse(open(os.path.join(ROOT, "synthetic", "__init__.py"), encoding="utf-8").read())
    if ast.get_docstring(tree) is not None:
        tree.body = tree.body[1:]                   # the module docstring describes the rule itself
    text = ast.unparse(tree)                        # code only: comments dropped
    for pat in (r"\b448\b", r"float8", r"e4m3", r"amax", r"\bscale_from", r"quant"):
        assert not re.search(pat, text, re.IGNORECASE), pat
