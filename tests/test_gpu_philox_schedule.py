"""GPU parity of the Philox uniforms and the schedule kernel (through the C
ABI) against the oracle: bit-exact, apart from survival products within
1e-6 of tau."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_93_b200 as sv
from _parity import SCHEDULE_TIE, gpu_schedule

pytestmark = pytest.mark.gpu


def test_philox_raw_blocks_bit_exact():
    rng = np.random.default_rng(0)
    n = 4096
    ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 2**32, size=(n, 2), dtype=np.uint64).astype(np.uint32)
    ctr[:4] = [[0, 0, 0, 0], [2**32 - 1] * 4, [1, 2, 3, 4], [7, 0, 1, 0]]
    key[:4] = [[0, 0], [2**32 - 1] * 2, [5, 6], [0, 0]]
    to = lambda a: torch.from_numpy(a.view(np.int32)).cuda()
    out = torch.zeros(n, 4, dtype=torch.int32, device="cuda")
    sv.sv_philox4x32_10(to(ctr), to(key), out)
    got = out.cpu().numpy().view(np.uint32)
    for k in range(n):
        np.testing.assert_array_equal(got[k], oracle.philox4x32_10(ctr[k], key[k]))


@pytest.mark.parametrize("seed", [0, 1, 0xDEADBEEF, 2**64 - 1])
def test_uniforms_bit_exact(seed):
    rng = np.random.default_rng(seed & 0xFFFF)
    n = 200_000
    row = rng.integers(0, 2**40, size=n, dtype=np.int64)
    row[:3] = [0, 1, 2**32 + 5]
    pos = rng.integers(0, 64, size=n).astype(np.int32)
    draw = rng.integers(0, 2, size=n).astype(np.int32)
    out = torch.zeros(n, dtype=torch.float32, device="cuda")
    sv.sv_philox_uniforms(seed, torch.from_numpy(row).cuda(), torch.from_numpy(pos).cuda(),
                          torch.from_numpy(draw).cuda(), out)
    want = oracle.uniform_batch(seed, row.astype(np.uint64), pos.astype(np.uint32),
                                draw.astype(np.uint32))
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64), want)


@pytest.mark.parametrize("B,K", [(1, 1), (256, 8), (512, 16), (3000, 64)])
@pytest.mark.parametrize("beta", [(8.0, 2.0), (6.0, 3.0), (50.0, 1.0)])
def test_schedule_matches_oracle(B, K, beta):
    rng = np.random.default_rng(B + K)
    conf = rng.beta(beta[0], beta[1], size=(B, K)).astype(np.float32)
    conf[0, 0] = np.nan if B > 1 else conf[0, 0]
    if B > 4:
        conf[1, :] = 1.0
        conf[2, 0] = -0.5
        conf[3, 1] = 1.7
    c = torch.from_numpy(conf).cuda()
    for tau in (-0.1, 0.0, 0.1, 0.3, 0.6, 0.999, 1.0, 1.01):
        g = gpu_schedule(c, tau).cpu().numpy()
        want, S, _ = oracle.schedule(conf, tau)
        tie = np.any(np.abs(S - tau) < SCHEDULE_TIE, axis=1)
        assert np.array_equal(g[~tie], want[~tie]), tau
        assert np.all((g >= 0) & (g <= K))
