"""Pins for the oracle's per-position temperature scaling of the confidence
head (umans.ai page, "What DSpark adds", item "2. Verify smarter": one
temperature for each draft position, chosen on blocks kept aside; zhichai.net topic, "Under
the hood": Sequential Temperature Scaling).

Each pin comes from outside the oracle's code: a closed form for a constant
logit, a brute-force minimisation of the likelihood written here with
numpy, exact invariances, hand-computed calibration errors, and recovery of
a planted temperature from synthetic data drawn with it."""
import math

import numpy as np
import pytest

import oracle


def _blocks(survived, K=1):
    """Accepted lengths for K = 1 blocks: a = 1 if the token survived."""
    return np.asarray(survived, dtype=np.int32)


@pytest.mark.parametrize("c,p", [(2.0, 0.7), (0.5, 0.9), (-1.5, 0.3), (3.0, 0.55)])
def test_constant_logit_closed_form(c, p):
    # Every observed logit equal to c, a fraction p survived: the likelihood
    # is maximised where sigmoid(c / T) = p, i.e. T = c / logit(p).
    n = 1000
    k = int(round(p * n))
    a = _blocks([1] * k + [0] * (n - k))
    l = np.full((n, 1), c, np.float32)
    T, _, cnt = oracle.sts_fit(l, a)
    want = float(np.float32(c)) / math.log((k / n) / (1 - k / n))
    assert cnt == n
    assert abs(T[0] - want) <= 1e-12 * abs(want)


def _nll(beta, l, s):
    return float(np.sum(np.logaddexp(0.0, -s * beta * l)))


def _brute_force_T(l, s, tmin=1e-2, tmax=1e2):
    """argmin of the NLL over beta in [1/tmax, 1/tmin]: a dense log grid,
    then golden-section search around the best grid point."""
    betas = np.exp(np.linspace(np.log(1 / tmax), np.log(1 / tmin), 4001))
    vals = np.array([_nll(b, l, s) for b in betas])
    j = int(np.argmin(vals))
    lo, hi = betas[max(j - 1, 0)], betas[min(j + 1, len(betas) - 1)]
    g = (math.sqrt(5) - 1) / 2
    for _ in range(200):
        x1, x2 = hi - g * (hi - lo), lo + g * (hi - lo)
        if _nll(x1, l, s) < _nll(x2, l, s):
            hi = x2
        else:
            lo = x1
    return 1.0 / (0.5 * (lo + hi))


def test_brute_force_minimiser():
    rng = np.random.default_rng(7)
    N, K = 3000, 3
    l = rng.normal(0.8, 2.0, size=(N, K)).astype(np.float32)
    a = rng.integers(0, K + 1, size=N).astype(np.int32)
    T, _, _ = oracle.sts_fit(l, a)
    for i in range(K):
        obs = a >= i
        s = np.where(a[obs] > i, 1.0, -1.0)
        want = _brute_force_T(l[obs, i].astype(np.float64), s)
        # golden-section search on likelihood values resolves the minimiser
        # only to about sqrt(eps) of a flat optimum
        assert abs(T[i] - want) <= 1e-5 * want, (i, T[i], want)


def test_scale_and_flip_invariance():
    rng = np.random.default_rng(3)
    N = 5000
    l = rng.normal(1.0, 1.5, size=(N, 1)).astype(np.float32)
    a = (rng.random(N) < 0.6).astype(np.int32)
    T, _, _ = oracle.sts_fit(l, a)
    # scaling the logits by a power of two scales T exactly
    T2, _, _ = oracle.sts_fit(l * 4, a)
    assert abs(T2[0] - 4 * T[0]) <= 1e-12 * T2[0]
    # negating the logits and flipping every outcome leaves T unchanged
    T3, _, _ = oracle.sts_fit(-l, 1 - a)
    assert abs(T3[0] - T[0]) <= 1e-12 * T[0]


def test_only_blocks_that_reached_the_position_count():
    rng = np.random.default_rng(11)
    N, K = 4000, 4
    l = rng.normal(1.0, 1.0, size=(N, K)).astype(np.float32)
    a = rng.integers(0, K + 1, size=N).astype(np.int32)
    T, _, cnt = oracle.sts_fit(l, a)
    # logits of positions a block never reached must not matter
    l2 = l.copy()
    for n in range(N):
        l2[n, a[n] + 1:] = rng.normal(0.0, 50.0, size=max(0, K - a[n] - 1))
    T2, _, cnt2 = oracle.sts_fit(l2, a)
    np.testing.assert_array_equal(T, T2)
    assert cnt == cnt2 == int(np.minimum(a + 1, K).sum())
    # skipped blocks (a < 0) contribute nothing
    T3, _, cnt3 = oracle.sts_fit(np.vstack([l, l[:10] * 9]), np.concatenate([a, -np.ones(10, np.int32)]))
    np.testing.assert_array_equal(T, T3)
    assert cnt3 == cnt


def test_degenerate_positions():
    # no block reaches position 2 -> T = 1; every logit 0 -> flat -> T = 1
    l = np.array([[1.0, 2.0, 3.0], [0.5, 1.0, 2.0]], np.float32)
    a = np.array([1, 0], np.int32)
    T, _, _ = oracle.sts_fit(l, a)
    assert T[2] == 1.0
    T, _, _ = oracle.sts_fit(np.zeros((6, 2), np.float32), np.array([0, 1, 2, 2, 1, 0], np.int32))
    assert list(T) == [1.0, 1.0]
    # all survive with positive logits: the likelihood keeps rising with
    # confidence, so T goes to the lower end; all fail: to the upper end
    l = np.full((50, 1), 1.0, np.float32)
    T, _, _ = oracle.sts_fit(l, np.ones(50, np.int32), tmin=0.05, tmax=20.0)
    assert T[0] == pytest.approx(0.05, rel=1e-15)
    T, _, _ = oracle.sts_fit(l, np.zeros(50, np.int32), tmin=0.05, tmax=20.0)
    assert T[0] == pytest.approx(20.0, rel=1e-15)


def test_ece_hand_worked():
    # four blocks at confidence 0.5 (bin 7), three survive:
    # |3 - 4 * 0.5| / 4 = 0.25; the fit leaves l = 0 at T = 1
    l = np.zeros((4, 1), np.float32)
    T, ece, _ = oracle.sts_fit(l, np.array([1, 1, 1, 0], np.int32))
    assert ece[0] == pytest.approx(0.25, abs=1e-15)
    assert ece[1] == pytest.approx(0.25, abs=1e-15)
    # ten blocks at confidence 0.8 with eight survivors: calibrated, ECE 0,
    # and the fit keeps T = 1 (sigmoid(l / T) = 0.8 at T = 1)
    c = math.log(0.8 / 0.2)
    l = np.full((10, 1), c, np.float32)
    a = np.array([1] * 8 + [0] * 2, np.int32)
    T, ece, _ = oracle.sts_fit(l, a)
    assert T[0] == pytest.approx(float(np.float32(c)) / c, rel=1e-9)
    assert ece[0] == pytest.approx(abs(8 - 10 * (1 / (1 + math.exp(-float(np.float32(c)))))) / 10,
                                   abs=1e-12)
    # two bins: confidences 0.2 (1 of 2 survive) and 0.9 (2 of 2)
    l = np.array([[math.log(0.25)], [math.log(0.25)], [math.log(9.0)], [math.log(9.0)]],
                 np.float32)
    a = np.array([1, 0, 1, 1], np.int32)
    conf = 1 / (1 + np.exp(-l[:, 0].astype(np.float64)))
    want = (abs(1 - conf[0] - conf[1]) + abs(2 - conf[2] - conf[3])) / 4
    _, ece, _ = oracle.sts_fit(l, a)
    assert ece[0] == pytest.approx(want, abs=1e-12)


def test_recovers_planted_temperature():
    # Survival drawn from sigmoid(l*) along the block; the head reports
    # l = kappa_i * l* (overconfident for kappa > 1).  The fitted T_i must
    # recover kappa_i, and calibration must improve.
    rng = np.random.default_rng(2024)
    N, K = 200000, 4
    lstar = rng.normal(1.8, 1.0, size=(N, K))
    kappa = np.array([1.25, 1.5, 1.75, 2.0])
    l = (lstar * kappa).astype(np.float32)
    y = rng.random((N, K)) < 1 / (1 + np.exp(-lstar))
    a = np.where(y.all(1), K, np.argmin(y, axis=1)).astype(np.int32)
    T, ece, _ = oracle.sts_fit(l, a)
    np.testing.assert_allclose(T, kappa, rtol=0.03)
    assert ece[0] > 0.03 and ece[1] < 0.01
