"""The product path and the oracle stay apart, and the product has no
fallback: importing the package pulls in no oracle code, neither side names
the other in its sources, and without the CUDA library (or with CPU tensors)
every call raises instead of computing."""
import os
import re
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_attention_coarse_b200")


def sources(top, exts):
    for dirpath, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_importing_the_package_loads_no_oracle():
    code = ("import sys, block_sparse_attention_coarse_b200, block_sparse_attention_coarse_b200.shard; "
            "print(sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "[]"


def test_product_sources_do_not_name_the_oracle():
    pat = re.compile(r"^\s*(import|from)\s+oracle\b|#include\s+[\"<][^\">]*oracle|isa_oracle", re.M)
    for path in sources(PKG, (".py", ".cu", ".cuh", ".h")):
        assert not pat.search(open(path, encoding="utf-8").read()), path
    for path in sources(os.path.join(ROOT, "include"), (".h",)):
        assert "oracle" not in open(path, encoding="utf-8").read(), path


def test_oracle_sources_do_not_name_the_product():
    for path in sources(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        text = open(path, encoding="utf-8").read()
        assert "block_sparse_attention_coarse_b200" not in text and "libisa" not in text, path


def test_input_generators_hold_neither_side():
    """The seeded generators are the one module both sides use; they import
    neither the oracle nor the product."""
    pat = re.compile(r"^\s*(import|from)\s+(oracle|block_sparse_attention_coarse_b200)\b", re.M)
    for path in sources(os.path.join(ROOT, "workloads"), (".py",)):
        assert not pat.search(open(path, encoding="utf-8").read()), path


def test_missing_library_fails_loudly(monkeypatch):
    import block_sparse_attention_coarse_b200 as isa
    monkeypatch.setattr(isa, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libisa.so"))
    monkeypatch.setattr(isa, "_lib", None)
    p = isa.make_params(1, 1, 64, 64, 64)
    with pytest.raises(isa.IsaError, match="missing"):
        isa.workspace_size(p)


def test_cpu_tensors_are_refused():
    import block_sparse_attention_coarse_b200 as isa
    p = isa.make_params(1, 1, 64, 64, 64)
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    for call in (lambda: isa.plan(q, q, q, p), lambda: isa.dense(q, q, q, p),
                 lambda: isa.rope(q, q, p)):
        with pytest.raises(isa.IsaError, match="CUDA"):
            call()
