"""Parity at the full workload sizes, in the launch configuration the
benchmark times (same entry points, same workspace sizing).  Every row of
every workload is checked against the oracle: each must be bit-exact or one
of the oracle's tie-window outcomes.  The schedule is computed
independently on each side; a row whose survival product sits within 1e-6
of tau may take either length."""
import numpy as np
import pytest

import oracle
from speculative_decoding_verification_93_b200 import workloads
from _parity import SCHEDULE_TIE, check_batch, check_structure, gpu_schedule, gpu_verify

pytestmark = pytest.mark.gpu


def run_config(name, tau=None, seed=0):
    b = workloads.make_batch(name, device="cuda", tau=tau)
    if b.lengths is None:
        ln_gpu = gpu_schedule(b.conf, b.tau)
        ln_or, S, _ = oracle.schedule(b.conf.cpu().numpy(), b.tau)
        sched_tie = np.any(np.abs(S - b.tau) < SCHEDULE_TIE, axis=1)
        assert np.array_equal(ln_gpu.cpu().numpy()[~sched_tie], ln_or[~sched_tie])
    else:
        ln_gpu = b.lengths
    g = gpu_verify(b.zt, b.zd, b.tokens, ln_gpu, b.temperature, seed)
    check_structure(g, b.tokens.cpu().numpy(), ln_gpu.cpu().numpy())
    assert g["status"] == 0
    res = check_batch(b, ln_gpu, g, seed)
    assert res["invalid"] == 0 and res["rows"] == b.spec.B
    # The fp32 kernels sit far inside the windows: rows that differ from the
    # oracle's own result (all of them inside a window) stay rare.
    assert res["window_valid"] <= max(2, res["rows"] // 50), res
    return res


def test_c1_full():
    print(run_config("c1"))


def test_c2_full():
    print(run_config("c2"))


def test_c3_full():
    print(run_config("c3"))


@pytest.mark.parametrize("tau", [0.1, 0.3, 0.6])
def test_c4_full(tau):
    print(run_config("c4", tau=tau))


@pytest.mark.parametrize("seed", [1, 2])
def test_c2_more_seeds(seed):
    print(run_config("c2", seed=seed))
