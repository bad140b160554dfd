"""GPU parity of the confidence head's per-position temperature scaling
(sv_sts_fit, sv_sts_apply) through the C ABI against the oracle, on seeded
synthetic held-out blocks.  Both sides sum in fp64; the GPU takes
safeguarded Newton steps where the oracle bisects, so the temperatures agree
to the fp32 rounding of the output."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200.workloads import sts_heldout

pytestmark = pytest.mark.gpu


def gpu_fit(l, a, tmin=1e-2, tmax=1e2):
    lt = torch.from_numpy(np.ascontiguousarray(l)).cuda()
    at = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    T = torch.full((l.shape[1],), -1.0, dtype=torch.float32, device="cuda")
    ece = torch.full((2,), -1.0, dtype=torch.float32, device="cuda")
    sv.sv_sts_fit(lt, at, T, ece, tmin=tmin, tmax=tmax)
    torch.cuda.synchronize()
    return T.cpu().numpy().astype(np.float64), ece.cpu().numpy().astype(np.float64)


def check(l, a, tmin=1e-2, tmax=1e2):
    Tg, eg = gpu_fit(l, a, tmin, tmax)
    To, eo, _ = oracle.sts_fit(l, a, tmin, tmax)
    np.testing.assert_allclose(Tg, To.astype(np.float32), rtol=3e-7, atol=0)
    np.testing.assert_allclose(eg, np.array(eo, np.float32), rtol=2e-6, atol=1e-7)
    return Tg, eg


@pytest.mark.parametrize("N,K,seed", [(1, 1, 0), (100, 3, 1), (2048, 8, 2), (2049, 8, 3),
                                      (50000, 8, 4), (262144, 8, 5), (9000, 64, 6)])
def test_sts_matches_oracle(N, K, seed):
    l, a = sts_heldout(N, K, seed=seed)
    check(l, a)


def test_sts_recovers_planted_overconfidence():
    l, a = sts_heldout(262144, 6, seed=11, kappa=(1.2, 2.0))
    T, ece = check(l, a)
    np.testing.assert_allclose(T, np.linspace(1.2, 2.0, 6), rtol=0.05)
    assert ece[0] > 0.03 and ece[1] < 0.01


def test_sts_degenerate_cases():
    rng = np.random.default_rng(5)
    N, K = 5000, 4
    l = rng.normal(1.0, 1.0, size=(N, K)).astype(np.float32)
    a = rng.integers(-1, 3, size=N).astype(np.int32)      # nobody reaches position 3
    T, _ = check(l, a)
    assert T[3] == 1.0
    l0 = np.zeros((N, K), np.float32)                      # flat likelihood
    T, _ = check(l0, rng.integers(0, K + 1, size=N).astype(np.int32))
    assert list(T) == [1.0] * K
    lp = np.abs(l) + 0.1                                   # all survive / all fail
    T, _ = check(lp, np.full(N, K, np.int32), tmin=0.05, tmax=20.0)
    np.testing.assert_allclose(T, 0.05, rtol=1e-7)
    T, _ = check(lp, np.zeros(N, np.int32), tmin=0.05, tmax=20.0)
    assert T[0] == pytest.approx(20.0, rel=1e-7)


def test_sts_apply():
    l, a = sts_heldout(3000, 5, seed=9)
    T = np.array([0.7, 1.0, 1.3, 2.0, 5.0], np.float32)
    out = torch.empty(l.shape, dtype=torch.float32, device="cuda")
    sv.sv_sts_apply(torch.from_numpy(l).cuda(), torch.from_numpy(T).cuda(), out)
    torch.cuda.synchronize()
    want = 1.0 / (1.0 + np.exp(-(l.astype(np.float64) / T.astype(np.float64))))
    np.testing.assert_allclose(out.cpu().numpy(), want, rtol=2e-6, atol=1e-7)


def test_barrier_wait_that_runs_out_returns_nan():
    """The grid barrier's wait is bounded in wall time.  With the bound set
    near zero (a test export), the CTAs that arrive early give up at once:
    the call returns, the temperatures come out NaN, the ECE output is not
    written, and the expired waits are counted.  Nothing hangs or faults,
    and with the bound restored the same fit matches the oracle again."""
    l, a = sts_heldout(8192, 4, seed=13)      # 4 chunks x 4 positions: 16 CTAs
    sv.sv_debug_sts_timeouts()                # clear the count
    outcomes = []
    try:
        sv.sv_debug_sts_wait_limit(1)
        for _ in range(3):
            T, ece = gpu_fit(l, a)
            outcomes.append((sv.sv_debug_sts_timeouts(), T, ece))
    finally:
        sv.sv_debug_sts_wait_limit(0)         # back to the 1 s default
    timed_out = [o for o in outcomes if o[0] > 0]
    assert timed_out, [o[0] for o in outcomes]
    for n, T, ece in timed_out:
        assert np.all(np.isnan(T)), T
        assert list(ece) == [-1.0, -1.0]      # left as the caller filled it
    for n, T, ece in outcomes:
        if n == 0:                            # a fit whose barriers all met in time
            assert np.all(np.isfinite(T))
    check(l, a)
    assert sv.sv_debug_sts_timeouts() == 0
