"""CPU checks of bench.py's pure helpers: the byte counts the roofline is
built on, and the code hash that decides whether a committed ncu capture
still describes the kernel."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_scheduled_bytes_by_hand():
    # rows: (L, T) = (4, 1.0), (0, 0.6), (3, 0.0); V = 10, bf16
    # target vectors 5 + 1 + 4 = 10, draft vectors 4 + 0 + 0 = 4 -> 14 * 20 B
    L = np.array([4, 0, 3])
    T = np.array([1.0, 0.6, 0.0])
    assert bench.scheduled_bytes(L, T, 10, 2) == 14 * 20
    # greedy drafter: no draft vectors
    assert bench.scheduled_bytes(L, T, 10, 2, has_draft=False) == 10 * 20


def test_needed_bytes_by_hand():
    # a = 1 (rejected at 1 of L = 4, sampled): target 0..1, draft 0..1 -> 4
    # a = 0 = L (sampled, bonus at 0): target 0 -> 1
    # a = 3 = L (greedy): target 0..3 -> 4
    L = np.array([4, 0, 3])
    a = np.array([1, 0, 3])
    T = np.array([1.0, 0.6, 0.0])
    assert bench.needed_bytes(a, L, T, 10, 4) == 9 * 40
    # the needed bytes never exceed the scheduled ones, and equal them when
    # every draft is accepted
    assert bench.needed_bytes(a, L, T, 10, 4) <= bench.scheduled_bytes(L, T, 10, 4)
    assert bench.needed_bytes(L, L, T, 10, 4) == bench.scheduled_bytes(L, T, 10, 4)


def test_code_only_ignores_comments_and_layout_but_not_code():
    src = 'int a = 1; // one\n/* block\n comment */ asm("ld.global // not a comment");\n'
    assert bench.code_only(src) == 'inta=1;asm("ld.global // not a comment");'
    assert bench.code_only(src.replace("// one", "// uno")) == bench.code_only(src)
    assert bench.code_only(src.replace("a = 1", "a = 2")) != bench.code_only(src)
    assert bench.code_only("char c = '\\'';  // x") == "charc='\\'';"
