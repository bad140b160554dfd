"""Structural rules checked on the CPU: the CUDA path and the oracle share no
code and never import each other, the product fails loudly without its
library (there is no fallback), and the seeded input generators -- the one
module both sides use -- are deterministic."""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "speculative_decoding_verification_93_b200")


def _sources(folder, exts):
    for dirpath, _, files in os.walk(folder):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_product_never_imports_or_links_the_oracle():
    for p in _sources(PKG, (".py", ".cu", ".cuh", ".h")):
        text = open(p).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), p
        assert "liboracle" not in text and "oracle.c" not in text, p


def test_oracle_never_imports_the_product():
    for p in _sources(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        text = open(p).read()
        assert "speculative_decoding_verification_93_b200" not in text, p
        assert "libsv" not in text and "sv_device" not in text, p


def test_missing_library_fails_loudly(monkeypatch):
    from speculative_decoding_verification_93_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "libsv.so"))
    with pytest.raises(ImportError):
        _binding.lib()


def test_input_generators_are_deterministic():
    from speculative_decoding_verification_93_b200 import workloads
    a = workloads.make_batch("c0", device="cpu")
    b = workloads.make_batch("c0", device="cpu")
    for name in ("zt", "zd", "tokens", "temperature", "conf", "lengths"):
        x, y = getattr(a, name), getattr(b, name)
        assert (x is None) == (y is None)
        if x is not None:
            assert torch.equal(x, y), name
    assert tuple(a.zt.shape) == (4, 5, 1000) and a.zt.dtype == torch.float32
    s1 = workloads.random_small(8, 3, 50, dtype=torch.bfloat16, seed=4)
    s2 = workloads.random_small(8, 3, 50, dtype=torch.bfloat16, seed=4)
    s3 = workloads.random_small(8, 3, 50, dtype=torch.bfloat16, seed=5)
    assert torch.equal(s1.zt, s2.zt) and torch.equal(s1.tokens, s2.tokens)
    assert not torch.equal(s1.zt, s3.zt)
    l1, a1 = workloads.sts_heldout(1000, 4, seed=2)
    l2, a2 = workloads.sts_heldout(1000, 4, seed=2)
    assert np.array_equal(l1, l2) and np.array_equal(a1, a2)
