"""GPU parity of sv_schedule_admit (hardware-aware admission) through the C
ABI against the oracle: identical lengths, admitted count and threshold.
Survivals are fp64 on both sides in the same order, so the sort keys agree
bit for bit; only the partial sums run in a different order."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_93_b200 as sv

pytestmark = pytest.mark.gpu


def run_gpu(conf, speed):
    c = torch.from_numpy(conf).cuda()
    s = torch.from_numpy(speed).cuda()
    ln = torch.full((conf.shape[0],), -7, dtype=torch.int32, device="cuda")
    tau = torch.zeros(1, dtype=torch.float32, device="cuda")
    sv.sv_schedule_admit(c, s, ln, tau)
    torch.cuda.synchronize()
    return ln.cpu().numpy(), float(tau.item())


def tables(B, K):
    n = np.arange(B * (K + 1) + 2, dtype=np.float64)
    out = []
    for n0 in (3.0, 30.0, 300.0, 3000.0):
        out.append((1000.0 / (1.0 + n / n0)).astype(np.float32))
    knee = max(B, 1) * 2
    out.append(np.where(n < knee, 500.0, 500.0 * knee / np.maximum(n, 1)).astype(np.float32))
    out.append(np.full(n.size, 7.0, np.float32))                       # flat: admit all
    out.append((1000.0 / (1.0 + n / 50.0))[: B + max(1, B * K // 3)].astype(np.float32))  # short
    return out


@pytest.mark.parametrize("B,K", [(4, 4), (100, 7), (256, 8), (512, 16), (1024, 8), (8192, 1)])
def test_admission_matches_oracle(B, K):
    rng = np.random.default_rng(B * 31 + K)
    for conf in (rng.beta(8, 2, size=(B, K)).astype(np.float32),
                 rng.beta(6, 3, size=(B, K)).astype(np.float32)):
        for speed in tables(B, K):
            ln_g, tau_g = run_gpu(conf, speed)
            ln_o, tau_o, k_o, _ = oracle.schedule_admit(conf, speed)
            assert np.array_equal(ln_g, ln_o), (B, K, int(ln_g.sum()), k_o)
            assert ln_g.sum() == k_o
            assert tau_g == np.float32(tau_o)


def test_admission_ties_nan_and_clamps():
    B, K = 300, 6
    rng = np.random.default_rng(5)
    row = rng.beta(8, 2, size=K).astype(np.float32)
    conf = np.tile(row, (B, 1))                     # every row ties with every other
    conf[7] = np.nan
    conf[8, 2] = -1.0
    conf[9, 0] = 2.5
    for speed in tables(B, K):
        ln_g, tau_g = run_gpu(conf, speed)
        ln_o, tau_o, k_o, _ = oracle.schedule_admit(conf, speed)
        assert np.array_equal(ln_g, ln_o)
        assert tau_g == np.float32(tau_o)
