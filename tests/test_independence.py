"""The oracle and the CUDA path share no code: neither imports, includes or links
the other, and the product package never touches the oracle."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "exact_attention_103_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        if "_build" in dirpath or "__pycache__" in dirpath:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def test_product_package_never_touches_the_oracle():
    for path in _files(PKG, (".py", ".cu", ".cuh", ".h", ".c")):
        text = open(path, encoding="utf-8").read()
        assert not re.search(r"import oracle|from oracle|attn_oracle|liboracle", text), path


def test_oracle_uses_nothing_of_the_cuda_path():
    for path in _files(ORACLE, (".py", ".c", ".h")):
        text = open(path, encoding="utf-8").read()
        assert "exact_attention_103_b200" not in text, path
        assert "libattn" not in text, path
        assert not re.search(r'#include\s+"', text), path  # system headers only


def test_shared_input_module_holds_no_attention_arithmetic():
    text = open(os.path.join(ROOT, "attn_inputs.py"), encoding="utf-8").read()
    for word in ("softmax", "exp(", "exp2", "logsumexp", "matmul", " @ ", "einsum"):
        assert word not in text, word
