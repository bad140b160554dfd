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


def test_committed_traffic_needs_the_current_kernel_hash(tmp_path, monkeypatch):
    p = tmp_path / "t.json"
    p.write_text('{"kernel_source_hash": "%s", "workloads": {"c2": '
                 '{"dram_bytes_per_launch": 123}}}' % bench.kernel_hash())
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
    assert bench.committed_traffic("c2") == 123.0
    assert bench.committed_traffic("c3") is None
    p.write_text('{"kernel_source_hash": "0000", "workloads": {"c2": '
                 '{"dram_bytes_per_launch": 123}}}')
    assert bench.committed_traffic("c2") is None


def test_l2_flush_only_for_inputs_near_the_l2_size():
    from types import SimpleNamespace
    import torch
    small = SimpleNamespace(zt=torch.empty(4, 5, 1000), zd=torch.empty(4, 4, 1000))
    big = SimpleNamespace(zt=torch.empty(1, 1, 1), zd=torch.empty(1, 1, 1))
    big.zt = SimpleNamespace(numel=lambda: 64 * 5 * 129280)
    big.zd = SimpleNamespace(numel=lambda: 64 * 4 * 129280)
    assert bench.needs_flush(small, 4)            # c0: 0.14 MB
    assert bench.needs_flush(big, 2)              # c1: 149 MB < 252 MB
    big.zt = SimpleNamespace(numel=lambda: 256 * 9 * 129280)
    big.zd = SimpleNamespace(numel=lambda: 256 * 8 * 129280)
    assert not bench.needs_flush(big, 2)          # c2: 1.1 GB
