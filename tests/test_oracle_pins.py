"""Further pins for the oracle: greedy reduction, closed-form acceptance,
chi-square of Philox-keyed draws, the schedule's worked example and
invariants, softmax statistics in closed form and the data checks."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy import stats as sst

import oracle
from speculative_decoding_verification_93_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def softmax(z, T):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


# --------------------------------------------------------------------------
# Greedy verification (T = 0)
# --------------------------------------------------------------------------

def brute_force_greedy(zt, x, L):
    a = 0
    while a < L and x[a] == int(np.argmax(zt[a])):   # numpy: first max wins
        a += 1
    return a, [int(t) for t in x[:a]] + [int(np.argmax(zt[a]))]


def test_greedy_is_longest_matching_prefix_with_ties():
    rng = np.random.default_rng(0)
    B, K, V = 300, 5, 7
    zt = rng.integers(-2, 3, size=(B, K + 1, V)).astype(np.float32)   # many ties
    zd = rng.integers(-2, 3, size=(B, K, V)).astype(np.float32)
    # drafts: half agree with the target argmax, half random
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    agree = rng.random((B, K)) < 0.7
    x = np.where(agree, zt[:, :K].argmax(-1), x).astype(np.int32)
    L = rng.integers(0, K + 1, size=B).astype(np.int32)
    T = np.zeros(B, dtype=np.float32)
    out, acc, diag, st = oracle.verify(zt, zd, x, L, T, seed=9)
    assert st == 0
    for b in range(B):
        a, toks = brute_force_greedy(zt[b], x[b], L[b])
        assert acc[b] == a
        assert list(out[b, :a + 1]) == toks
        assert np.all(out[b, a + 1:] == -1)


def test_greedy_equals_sampling_path_with_one_hot_target():
    """With logits spaced >= 1 apart and T = 1e-3, p and q are one-hot in fp64;
    the sampling rule then reduces to greedy verification whatever the
    uniforms (draft = drafter's argmax)."""
    rng = np.random.default_rng(1)
    B, K, V = 200, 4, 9
    zt = np.stack([np.stack([rng.permutation(V) for _ in range(K + 1)]) for _ in range(B)])
    zd = np.stack([np.stack([rng.permutation(V) for _ in range(K)]) for _ in range(B)])
    # make drafts agree with the target often
    flip = rng.random((B, K)) < 0.6
    zd = np.where(flip[..., None], zt[:, :K], zd)
    zt = zt.astype(np.float32)
    zd = zd.astype(np.float32)
    x = zd.argmax(-1).astype(np.int32)
    L = rng.integers(0, K + 1, size=B).astype(np.int32)
    g_out, g_acc, _, _ = oracle.verify(zt, zd, x, L, np.zeros(B, np.float32), seed=3)
    s_out, s_acc, _, _ = oracle.verify(zt, zd, x, L, np.full(B, 1e-3, np.float32), seed=3)
    np.testing.assert_array_equal(g_acc, s_acc)
    np.testing.assert_array_equal(g_out, s_out)


# --------------------------------------------------------------------------
# Sampling: closed form and chi-square with the Philox uniforms
# --------------------------------------------------------------------------

def _identical_rows(V, K, T, B, seed, noise=1.0, std=2.0):
    g = torch.Generator().manual_seed(seed)
    zt1 = torch.randn(1, K + 1, V, generator=g) * std
    zd1 = zt1[:, :K] + noise * torch.randn(1, K, V, generator=g)
    zt = zt1.expand(B, K + 1, V).contiguous()
    zd = zd1.expand(B, K, V).contiguous()
    temp = torch.full((B,), T)
    x = workloads.gumbel_tokens(zd, temp, g, rows_per_block=4096)
    return zt.numpy(), zd.numpy(), x.numpy(), temp.numpy()


def test_mean_accept_length_matches_closed_form():
    """E[a] = sum_{i=1..L} prod_{j<i} beta_j, beta_j = sum_v min(p_j, q_j)
    (drafts sampled from q, positions independent)."""
    V, K, T, B = 2000, 4, 1.0, 4000
    zt, zd, x, temp = _identical_rows(V, K, T, B, seed=5)
    L = np.full(B, K, np.int32)
    out, acc, _, st = oracle.verify(zt, zd, x, L, temp, seed=11)
    assert st == 0
    p = [softmax(zt[0, i], T) for i in range(K + 1)]
    q = [softmax(zd[0, i], T) for i in range(K)]
    beta = [np.minimum(p[i], q[i]).sum() for i in range(K)]
    Ea = sum(np.prod(beta[:i]) for i in range(1, K + 1))
    se = acc.std(ddof=1) / math.sqrt(B)
    assert abs(acc.mean() - Ea) < 4 * se, (acc.mean(), Ea, se)


@pytest.mark.parametrize("T", [0.6, 1.0])
def test_chi_square_of_emitted_tokens(T):
    V, K, B = 5, 2, 60000
    zt, zd, x, temp = _identical_rows(V, K, T, B, seed=21, noise=1.2, std=1.0)
    L = np.full(B, K, np.int32)
    out, acc, _, _ = oracle.verify(zt, zd, x, L, temp, seed=2024)
    for i in range(K + 1):
        sel = acc >= i
        counts = np.bincount(out[sel, i], minlength=V)
        expect = sel.sum() * softmax(zt[0, i], T)
        chi2 = ((counts - expect) ** 2 / expect).sum()
        assert sst.chi2.sf(chi2, V - 1) > 1e-3, (i, counts, expect)


def test_row_id_keys_the_uniforms():
    """Rows are keyed by their global id: verifying rows [8, 16) alone with
    row_base 8 (or explicit row ids) equals the same rows of the full run."""
    V, K, B = 50, 3, 16
    zt, zd, x, temp = _identical_rows(V, K, 1.0, B, seed=2)
    L = np.full(B, K, np.int32)
    full = oracle.verify(zt, zd, x, L, temp, seed=7)
    part = oracle.verify(zt[8:], zd[8:], x[8:], L[8:], temp[8:], seed=7, row_base=8)
    ids = oracle.verify(zt[8:], zd[8:], x[8:], L[8:], temp[8:], seed=7,
                        row_ids=np.arange(8, 16))
    for r in (part, ids):
        np.testing.assert_array_equal(full[0][8:], r[0])
        np.testing.assert_array_equal(full[1][8:], r[1])


# --------------------------------------------------------------------------
# Schedule
# --------------------------------------------------------------------------

def test_schedule_worked_examples():
    g = json.load(open(os.path.join(GOLDEN, "schedule_worked.json")))
    for case in g["cases"]:
        c = np.array([[float(v) for v in case["conf"]]], dtype=np.float32)
        for tau, want in case["tau_to_L"]:
            ln, S, _ = oracle.schedule(c, tau)
            assert ln[0] == want, (case["conf"], tau, ln[0])
            np.testing.assert_allclose(S[0], case["S"], rtol=1e-6, atol=1e-7)


def test_schedule_invariants():
    rng = np.random.default_rng(3)
    B, K = 500, 12
    conf = rng.beta(6, 3, size=(B, K)).astype(np.float32)
    taus = np.linspace(-0.1, 1.1, 61)
    prev = None
    for tau in taus:
        ln, S, _ = oracle.schedule(conf, tau)
        assert np.all(np.diff(S, axis=1) <= 0)             # survival never grows
        assert np.all((ln >= 0) & (ln <= K))
        if tau <= 0:
            assert np.all(ln == K)
        if tau > 1:
            assert np.all(ln == 0)
        # every kept prefix survives at >= tau, the next one does not
        for b in range(B):
            if ln[b] > 0:
                assert S[b, ln[b] - 1] >= tau
            if ln[b] < K:
                assert S[b, ln[b]] < tau
        if prev is not None:
            assert np.all(ln <= prev)                      # monotone in tau
        prev = ln


# --------------------------------------------------------------------------
# Softmax statistics and the data checks
# --------------------------------------------------------------------------

def test_stats_closed_forms():
    V = 37
    z = np.full((1, V), 1.25, np.float32)
    m, s, am = oracle.stats(z, 0.7)
    assert m[0] == 1.25 and abs(s[0] - V) < 1e-12 and am[0] == 0
    for T in (0.5, 1.0, 2.0):
        z = (-np.arange(V) * T * math.log(2.0)).astype(np.float64)
        zf = z.astype(np.float32)
        m, s, am = oracle.stats(zf[None], T)
        want = np.exp((zf.astype(np.float64) - zf.max()) / T).sum()
        assert abs(s[0] - want) < 1e-12 * want
        assert abs(s[0] - (2.0 - 2.0 ** (1 - V))) < 1e-6
        assert am[0] == 0 and m[0] == 0.0
    z = np.array([[1.0, 3.0, -1.0, 3.0]], np.float32)
    assert oracle.stats(z, 0.0)[2][0] == 1                  # first of the tied maxima


def test_bf16_widening_is_exact():
    vals = torch.tensor([1.0, -2.0, 0.15625, 3.0e38, -1e-30, float("inf"), float("-inf")],
                        dtype=torch.bfloat16)
    bits = vals.view(torch.int16).numpy().view(np.uint16)[None]
    m, _, am = oracle.stats(bits, 0.0)
    assert m[0] == float("inf") and am[0] == 5
    # the widened values must be the bf16 values themselves
    zt = np.concatenate([bits, bits])[None]                 # [1, 2, V]
    out, acc, _, _ = oracle.verify(zt, None, np.array([[5]], np.int32), [1],
                                   np.zeros(1, np.float32), seed=0)
    assert acc[0] == 1 and out[0, 1] == 5


def test_invalid_rows_are_marked_not_fatal():
    V, K = 10, 3
    zt = np.zeros((5, K + 1, V), np.float32)
    zd = np.zeros((5, K, V), np.float32)
    x = np.zeros((5, K), np.int32)
    x[1, 1] = V              # bad token inside the verified prefix
    x[4, 2] = -1             # bad token beyond L: ignored
    L = np.array([3, 3, 4, 1, 2], np.int32)   # row 2: length > K
    T = np.array([1.0, 1.0, 1.0, 5e-7, 1.0], np.float32)   # row 3: 0 < T < 1e-6
    out, acc, _, st = oracle.verify(zt, zd, x, L, T, seed=1)
    assert st == (1 | 2 | 4)
    assert list(acc[[1, 2, 3]]) == [-1, -1, -1]
    assert np.all(out[[1, 2, 3]] == -1)
    assert acc[0] >= 0 and acc[4] >= 0
    T2 = np.array([float("nan"), -1.0, float("inf"), 0.0, 1e-6], np.float32)
    out, acc, _, st = oracle.verify(zt, zd, np.zeros((5, K), np.int32), np.full(5, 2, np.int32),
                                    T2, seed=1)
    assert st == 4 and list(acc[:3]) == [-1, -1, -1] and acc[3] >= 0 and acc[4] >= 0


def test_verify_hand_worked_examples():
    """Hand-worked steps of the rule (tests/golden/verify_worked.json) with
    injected uniforms: accept/reject decisions, the residual and bonus
    inverse CDF on both sides of a boundary, temperature, L = 0, the greedy
    drafter and greedy ties."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "verify_worked.json")
    cases = json.load(open(path))["cases"]
    for c in cases:
        T = c["T"]
        if "logits" in c:
            zt = np.array(c["logits"], dtype=np.float64)
            zd = np.array(c["draft_logits"], dtype=np.float64)
        else:
            zt = T * np.log(np.array(c["p"], dtype=np.float64))
            zd = None if c.get("greedy_drafter") else T * np.log(np.array(c["q"], dtype=np.float64))
        K = zt.shape[0] - 1
        ua = np.zeros(K + 1)
        ur = np.zeros(K + 1)
        ua[:len(c["u_acc"])] = c["u_acc"]
        ur[:len(c["u_res"])] = c["u_res"]
        a, out, _ = oracle.verify_row_u(zt, zd, np.array(c["x"]), c["L"], T, ua, ur)
        assert a == c["accept"], c["name"]
        assert out.tolist() == c["tokens"], (c["name"], out.tolist())
