"""Pins for the oracle's hardware-aware admission (umans.ai page, "What DSpark
adds", item "2. Verify smarter"): a hand-worked example, closed forms for
two speed-table families, invariants, monotonicity in load, and agreement
with the threshold schedule at the admission threshold."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "admission_worked.json")))
    ln, tau, k, f = oracle.schedule_admit(np.array(g["conf"], np.float32),
                                          np.array(g["speed"], np.float32))
    assert k == g["admitted"]
    assert list(ln) == g["lengths"]
    assert abs(tau - g["tau"]) < 1e-6
    np.testing.assert_allclose(f[:len(g["f"])], g["f"], rtol=1e-6)


def test_constant_speed_admits_every_candidate_with_mass():
    rng = np.random.default_rng(0)
    conf = rng.beta(5, 2, size=(40, 6)).astype(np.float32)
    conf[3, 2] = 0.0                                # survival 0 from position 3 on
    speed = np.full(40 * 7 + 1, 10.0, np.float32)
    ln, tau, k, _ = oracle.schedule_admit(conf, speed)
    # every candidate with S > 0 raises E, and with flat speed f rises with E;
    # candidates are sorted, so admission stops at the first S == 0
    want = np.array([6] * 40)
    want[3] = 2
    assert k == want.sum() and np.array_equal(ln, want)


@pytest.mark.parametrize("n0", [5.0, 40.0, 300.0])
def test_hyperbolic_speed_closed_form(n0):
    """speed(n) = 1 / (n0 + n): candidate s is admitted iff it beats the
    current expected tokens per batch slot, s > E / (n0 + n)."""
    rng = np.random.default_rng(int(n0))
    B, K = 64, 8
    conf = rng.beta(6, 3, size=(B, K)).astype(np.float32)
    n = np.arange(B * (K + 1) + 1, dtype=np.float64)
    speed = (1.0 / (n0 + n)).astype(np.float32)
    ln, tau, k, _ = oracle.schedule_admit(conf, speed)
    # rebuild the sorted survivals independently (numpy cumprod on float64)
    S = np.cumprod(np.clip(conf.astype(np.float64), 0, 1), axis=1)
    order = sorted(range(B * K), key=lambda q: (-S.flat[q], q))
    E, nn, kk = float(B), B, 0
    for q in order:
        if not (S.flat[q] > E / (n0 + nn)):
            break
        E += S.flat[q]
        nn += 1
        kk += 1
    assert k == kk


def test_invariants_and_load_monotonicity():
    rng = np.random.default_rng(7)
    B, K = 128, 10
    conf = rng.beta(8, 2, size=(B, K)).astype(np.float32)
    n = np.arange(B * (K + 1) + 1, dtype=np.float64)
    prev = None
    for n0 in (2000.0, 800.0, 300.0, 100.0, 30.0, 5.0):       # heavier load -> steeper
        speed = (1000.0 / (1.0 + n / n0)).astype(np.float32)
        ln, tau, k, f = oracle.schedule_admit(conf, speed)
        assert ln.sum() == k and np.all((ln >= 0) & (ln <= K))
        assert np.all(np.diff(f[:k + 1]) > 0)                 # f rose at every admission
        if k < B * K and B + k + 1 < speed.size:
            assert f[k + 1] <= f[k]                            # ... and not at the stop
        if prev is not None:
            assert np.all(ln <= prev)                          # heavier load admits less
        prev = ln
        # with distinct survivals the admitted set is a threshold set
        ln_t, _, _ = oracle.schedule(conf, tau) if k > 0 else (np.zeros(B, np.int32), 0, 0)
        assert np.array_equal(ln_t, ln)


def test_table_limits_and_empty():
    conf = np.full((4, 3), 0.9, np.float32)
    ln, tau, k, _ = oracle.schedule_admit(conf, np.array([1, 1, 1, 1, 1, 1], np.float32))
    assert k == 1 and ln.sum() == 1          # batch of 4 fits; only n = 5 is in the table
    ln, tau, k, _ = oracle.schedule_admit(conf, np.array([1, 1, 1], np.float32))
    assert k == 0 and tau == float("inf") and ln.sum() == 0
