"""Parity at the full workload sizes, in the launch configuration the
benchmark times (same entry points, same workspace sizing).  Rows are
compared against the oracle in full where it finishes in seconds, else on
a seeded sample of rows (Philox is keyed by the global row id, so a sampled
row is computed exactly as in the full batch).  The schedule is computed
independently on each side; rows whose survival product sits within 1e-6 of
tau are excluded and counted."""
import numpy as np
import pytest

import oracle
from speculative_decoding_verification_93_b200 import workloads
from _parity import (SCHEDULE_TIE, check_structure, compare, gpu_schedule, gpu_verify,
                     oracle_verify)

pytestmark = pytest.mark.gpu


def run_config(name, tau=None, sample=None, seed=0):
    b = workloads.make_batch(name, device="cuda", tau=tau)
    B = b.spec.B
    if b.lengths is None:
        ln_gpu = gpu_schedule(b.conf, b.tau)
        ln_or, S, _ = oracle.schedule(b.conf.cpu().numpy(), b.tau)
        sched_tie = np.any(np.abs(S - b.tau) < SCHEDULE_TIE, axis=1)
        assert np.array_equal(ln_gpu.cpu().numpy()[~sched_tie], ln_or[~sched_tie])
    else:
        ln_gpu = b.lengths
        ln_or = b.lengths.cpu().numpy()
        sched_tie = np.zeros(B, dtype=bool)
    g = gpu_verify(b.zt, b.zd, b.tokens, ln_gpu, b.temperature, seed)
    check_structure(g, b.tokens.cpu().numpy(), ln_gpu.cpu().numpy())
    rows = None
    if sample is not None and sample < B:
        rows = np.sort(np.random.default_rng(7).choice(B, size=sample, replace=False))
    o = oracle_verify(b.zt, b.zd, b.tokens, ln_or, b.temperature, seed, rows=rows)
    ex = sched_tie if rows is None else sched_tie[rows]
    res = compare(g, o, rows=rows, extra_excluded=ex)
    res["sched_ties"] = int(sched_tie.sum())
    assert g["status"] == 0
    # rows inside a tie window are excluded from the bit-exact check and
    # counted; the fp32 kernels stay far inside the window, so rows that
    # actually differ must be rare even there
    assert res["tie_mismatches"] <= max(2, res["rows"] // 50), res
    return res


def test_c1_full():
    print(run_config("c1"))


def test_c2_full():
    print(run_config("c2"))


def test_c3_full():
    print(run_config("c3", sample=384))


@pytest.mark.parametrize("tau", [0.1, 0.3, 0.6])
def test_c4_sampled(tau):
    print(run_config("c4", tau=tau, sample=96))
