"""The oracle and the CUDA path share no code: neither includes, imports or
links the other, and the library's Python binding never reaches oracle/."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "quantized_expert_ffn_topk_b200")


def _files(d, exts):
    for base, _, names in os.walk(d):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(base, n)


def test_oracle_does_not_reach_the_library():
    for f in _files(os.path.join(ROOT, "oracle"), (".c", ".h", ".py")):
        src = open(f).read()
        assert "quantized_expert_ffn_topk_b200" not in src, f
        assert "moeq.h" not in src and "csrc" not in src, f
        assert not re.search(r"#include\s+\"\.\./", src), f


def test_library_does_not_reach_the_oracle():
    for f in _files(PKG, (".cu", ".cuh", ".h", ".c", ".cpp", ".py")):
        src = open(f).read()
        assert not re.search(r"\boracle\b", src), f
        assert "moe_ref_" not in src, f
        assert "synth" not in src, f


def test_generator_holds_no_method_arithmetic():
    for f in _files(os.path.join(ROOT, "synth"), (".c", ".h", ".cu", ".py")):
        src = open(f).read()
        for word in ("silu", "softmax", "rmsnorm", "moe_ref_", "moeq"):
            assert word not in src.lower(), (f, word)
