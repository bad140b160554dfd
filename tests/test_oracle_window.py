"""Pins for the oracle's tie-window outcome sets (``oracle.verify_window``).

A fp32 implementation may take a decision differently from the fp64 oracle
only when it lies within rounding of its threshold.  The window function
lists every outcome that such decisions can reach; the parity checks then
require each result to be one of them.  The function is pinned here by:

* hand-worked cases (``golden/window_worked.json``), each outcome set
  derived by hand from the rule (umans.ai "DeepSeek V4 Pro DSpark: the model
  isn't ready, the architecture is", section "Speculative decoding,
  briefly"; zhichai.net DSpark topic, section "Why LLMs speak so slowly");
* a brute-force restatement on tiny vocabularies, written here with numpy
  from the definitions (reachable accepted lengths from the accept
  thresholds; reachable tokens from the CDF intervals that meet the
  window), over random logits, uniforms and window widths, both drafters;
* zero windows reducing to the oracle's single outcome;
* the comparison module classifying planted results correctly.

It also pins the zero-residual fallback of the plain oracle, a branch only
rounding reaches.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import compare

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def softmax(z, T):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "window_worked.json")))["cases"],
                         ids=lambda c: c["name"])
def test_hand_worked_window_cases(case):
    T = case["T"]
    if "p" in case:
        zt = T * np.log(np.asarray(case["p"], dtype=np.float64))
        zd = T * np.log(np.asarray(case["q"], dtype=np.float64))
    else:
        zt = np.asarray(case["z_target"], dtype=np.float64)
        zd = np.asarray(case["z_draft"], dtype=np.float64)
    alt = oracle.verify_window_row_u(zt, zd, case["x"], case["L"], T, case["u_acc"],
                                     case["u_res"], case["w_acc"], case["w_cdf"])
    got = [list(map(int, r)) for r in alt if r[0] >= 0]
    assert got == case["outcomes"], (got, case["worked"])
    assert np.all(alt[len(got):] == -1)


def brute_force_outcomes(zt, zd, x, L, T, ua, ur, w_acc, w_cdf):
    """Outcome set from the definitions, in numpy: accepted length a is
    reachable iff every position before it can accept (u < acc, or within
    the window) and position a can reject (u >= acc, or within the window),
    or a == L; token v is reachable iff r(v) > 0 and its CDF interval
    [C(v-1), C(v)) meets the target window [max(0, u - w) R, (u + w) R] (a
    window past the total also reaches the last positive token)."""
    K = zt.shape[0] - 1
    V = zt.shape[1]
    p = [softmax(zt[i], T) for i in range(K + 1)]
    q = None if zd is None else [softmax(zd[i], T) for i in range(K)]

    def acc(i):
        qi = 1.0 if q is None else q[i][x[i]]
        if p[i][x[i]] == 0.0:
            return 0.0
        return min(1.0, p[i][x[i]] / qi)

    out = []
    for a in range(L + 1):
        can_reach = all((ua[i] < acc(i)) or abs(ua[i] - acc(i)) < w_acc for i in range(a))
        if not can_reach:
            break
        if a < L and not ((ua[a] >= acc(a)) or abs(ua[a] - acc(a)) < w_acc):
            continue
        if a < L:
            sub = np.zeros(V)
            if q is None:
                sub[x[a]] = 1.0
            else:
                sub = q[a]
            r = np.maximum(0.0, p[a] - sub)
            if r.sum() == 0.0:
                r = p[a]
        else:
            r = p[L]
        C = np.cumsum(r)
        R = C[-1]
        t0, t1 = max(0.0, ur[a] - w_cdf) * R, (ur[a] + w_cdf) * R
        reach = [v for v in range(V) if r[v] > 0 and (C[v - 1] if v else 0.0) <= t1 and C[v] > t0]
        if t1 >= R:
            reach.append(max(v for v in range(V) if r[v] > 0))
        t = ur[a] * R
        y = next((v for v in range(V) if C[v] > t), max(v for v in range(V) if r[v] > 0))
        out.append((a, y, min(reach), max(reach)))
    return out


@pytest.mark.parametrize("greedy_drafter", [False, True])
def test_window_sets_match_brute_force(greedy_drafter):
    rng = np.random.default_rng(11 + greedy_drafter)
    n_multi = n_span = 0
    for trial in range(1500):
        V = int(rng.integers(2, 7))
        K = int(rng.integers(1, 4))
        L = int(rng.integers(0, K + 1))
        T = float(rng.choice([0.6, 1.0, 1.7]))
        zt = rng.normal(0, 1.5, size=(K + 1, V))
        zd = None if greedy_drafter else zt[:K] + rng.normal(0, 1.0, size=(K, V))
        x = rng.integers(0, V, size=K).astype(np.int32)
        w_acc = float(rng.choice([0.0, 0.03, 0.15]))
        w_cdf = float(rng.choice([0.0, 0.03, 0.15]))
        ua = rng.random(K + 1)
        ur = rng.random(K + 1)
        alt = oracle.verify_window_row_u(zt, zd, x, L, T, ua, ur, w_acc, w_cdf)
        got = [tuple(int(v) for v in r) for r in alt if r[0] >= 0]
        want = brute_force_outcomes(zt, zd, x, L, T, ua, ur, w_acc, w_cdf)
        assert got == want, (trial, got, want)
        n_multi += len(got) > 1
        n_span += any(r[2] != r[3] for r in got)
    # the random cases exercise both kinds of window
    assert n_multi > 80 and n_span > 80


def test_zero_windows_reduce_to_the_oracle_result():
    rng = np.random.default_rng(5)
    for _ in range(300):
        V = int(rng.integers(1, 9))
        K = int(rng.integers(1, 5))
        L = int(rng.integers(0, K + 1))
        T = float(rng.choice([0.0, 0.5, 1.0]))
        zt = rng.normal(0, 2.0, size=(K + 1, V))
        zd = zt[:K] + rng.normal(0, 1.0, size=(K, V)) if rng.random() < 0.7 else None
        x = rng.integers(0, V, size=K).astype(np.int32)
        ua, ur = rng.random(K + 1), rng.random(K + 1)
        a, out, _ = oracle.verify_row_u(zt, zd, x, L, T, ua, ur)
        alt = oracle.verify_window_row_u(zt, zd, x, L, T, ua, ur, 0.0, 0.0)
        rows = [r for r in alt if r[0] >= 0]
        assert len(rows) == 1
        assert rows[0][0] == a and rows[0][1] == out[a] == rows[0][2] == rows[0][3]


def test_batch_window_matches_single_row():
    """The batch entry point (Philox uniforms, bf16 bits) lists the same
    outcomes as the single-row one given the same uniforms."""
    rng = np.random.default_rng(3)
    B, K, V = 12, 3, 40
    zt = (rng.normal(0, 2, size=(B, K + 1, V))).astype(np.float32)
    zd = (zt[:, :K] + rng.normal(0, 0.5, size=(B, K, V))).astype(np.float32)
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    L = rng.integers(0, K + 1, size=B).astype(np.int32)
    T = rng.choice([0.0, 0.7, 1.0], size=B).astype(np.float32)
    alt, st = oracle.verify_window(zt, zd, x, L, T, seed=77, w_acc=0.05, w_cdf=0.05)
    assert st == 0
    for b in range(B):
        ua = [oracle.uniform(77, b, i, 0) for i in range(K + 1)]
        ur = [oracle.uniform(77, b, i, 1) for i in range(K + 1)]
        one = oracle.verify_window_row_u(zt[b].astype(np.float64), zd[b].astype(np.float64),
                                         x[b], L[b], float(T[b]), ua, ur, 0.05, 0.05)
        assert np.array_equal(alt[b], one)


def test_zero_residual_falls_back_to_the_target():
    """p_0 and q_0 differ only below fp64 resolution at the draft token: the
    log-domain ratio is one ulp under 1, so a uniform of 1 - 2^-53 rejects,
    while every p - q rounds to <= 0.  The oracle then draws from p_0
    (flag 1) instead of failing: token 0 below the middle of p_0's CDF,
    token 1 above it, never the rejected draft through a fallback."""
    zt = np.array([[1e-16, 0.0], [0.0, 0.0]])
    zd = np.array([[0.0, 0.0]])
    x = np.array([1], dtype=np.int32)
    ua = np.array([1.0 - 2.0 ** -53, 0.0])
    for u, want in ((0.25, 0), (0.49, 0), (0.51, 1), (0.75, 1)):
        a, out, diag = oracle.verify_row_u(zt, zd, x, 1, 1.0, ua, np.array([u, 0.0]))
        assert a == 0 and out[0] == want and out[1] == -1
        assert diag[2] == 1.0            # zero-residual fallback, no CDF fallback
        assert abs(diag[4] - 1.0) < 1e-15  # drawn from p_0, total mass 1
        alt = oracle.verify_window_row_u(zt, zd, x, 1, 1.0, ua, np.array([u, 0.0]), 0.0, 0.0)
        assert list(alt[0]) == [0, want, want, want]


def _fetch_from(zt, zd):
    return lambda idx: (zt[idx], None if zd is None else zd[idx])


def test_compare_classifies_planted_results():
    """check_rows: the oracle's own result is bit-exact; a token moved within
    its draw window, or an accept decision flipped inside its window, is
    window-valid; a token moved outside the window, a wrong prefix or a wrong
    length is invalid."""
    rng = np.random.default_rng(21)
    B, K, V = 64, 4, 50
    zt = rng.normal(0, 1.0, size=(B, K + 1, V)).astype(np.float32)
    zd = (zt[:, :K] + rng.normal(0, 0.8, size=(B, K, V))).astype(np.float32)
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    L = np.full(B, K, dtype=np.int32)
    T = np.ones(B, dtype=np.float32)
    w = 0.02    # wide windows so that planted moves stay inside them
    o_tok, o_acc, _, _ = oracle.verify(zt, zd, x, L, T, 5)
    alt, _ = oracle.verify_window(zt, zd, x, L, T, 5, w_acc=w, w_cdf=w)
    fetch = _fetch_from(zt, zd)
    t = compare.check_rows(fetch, x, T, 5, L, L, L, L, o_tok, o_acc, w_acc=w, w_cdf=w)
    assert (t.rows, t.bit_exact, t.invalid) == (B, B, 0)
    g_tok, g_acc = o_tok.copy(), o_acc.copy()
    moved = flipped = 0
    for b in range(B):
        rows = [r for r in alt[b] if r[0] >= 0]
        own = [r for r in rows if r[0] == o_acc[b]][0]
        other = [r for r in rows if r[0] != o_acc[b]]
        if own[2] != own[3] and moved < 3:
            g_tok[b, own[0]] = own[3] if o_tok[b, own[0]] != own[3] else own[2]
            moved += 1
        elif other and flipped < 3:
            a2, y2 = other[0][0], other[0][1]
            g_acc[b] = a2
            g_tok[b] = -1
            g_tok[b, :a2] = x[b, :a2]
            g_tok[b, a2] = y2
            flipped += 1
    assert moved and flipped
    t = compare.check_rows(fetch, x, T, 5, L, L, L, L, g_tok, g_acc, w_acc=w, w_cdf=w)
    assert t.invalid == 0 and t.window_valid == moved + flipped
    # outside any window: a token past the span, a wrong prefix, a wrong length
    bad_tok = o_tok.copy()
    b0 = int(np.flatnonzero(o_acc < K)[0])
    span = [r for r in alt[b0] if r[0] == o_acc[b0]][0]
    bad_tok[b0, o_acc[b0]] = (span[3] + 5) % V if span[3] + 5 < V else span[2] - 5
    bad_pre = o_tok.copy()
    b1 = int(np.flatnonzero(o_acc > 0)[0])
    bad_pre[b1, 0] = (bad_pre[b1, 0] + 1) % V
    bad_len = L.copy()
    bad_len[2] = K - 1
    for tok, ln, want_row in ((bad_tok, L, b0), (bad_pre, L, b1), (o_tok, bad_len, 2)):
        t = compare.check_rows(fetch, x, T, 5, L, L, L, ln, tok, o_acc, w_acc=w, w_cdf=w)
        assert t.invalid >= 1 and want_row in t.invalid_rows


def test_schedule_span_and_alternative_lengths():
    """Rows whose survival product sits on tau may take either length; the
    comparison accepts a result verified at either one, and only those."""
    conf = np.array([[0.5, 0.5, 0.9], [0.9, 0.9, 0.9]], dtype=np.float32)
    L, lo, hi = compare.schedule_span(conf, 0.25)       # S = 0.5, 0.25, 0.225: tie at i = 2
    assert list(L) == [2, 3] and list(lo) == [1, 3] and list(hi) == [2, 3]
    rng = np.random.default_rng(2)
    B, K, V = 2, 3, 30
    zt = rng.normal(0, 1, size=(B, K + 1, V)).astype(np.float32)
    zd = (zt[:, :K] + rng.normal(0, 1, size=(B, K, V))).astype(np.float32)
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    T = np.ones(B, dtype=np.float32)
    alt_len = np.array([1, 3], dtype=np.int32)
    g_tok, g_acc, _, _ = oracle.verify(zt, zd, x, alt_len, T, 9)
    t = compare.check_rows(_fetch_from(zt, zd), x, T, 9, L, lo, hi, alt_len, g_tok, g_acc)
    assert t.invalid == 0 and t.schedule_window_rows == 1
    bad_len = np.array([0, 3], dtype=np.int32)
    b_tok, b_acc, _, _ = oracle.verify(zt, zd, x, bad_len, T, 9)
    t = compare.check_rows(_fetch_from(zt, zd), x, T, 9, L, lo, hi, bad_len, b_tok, b_acc)
    assert t.invalid == 1 and t.invalid_rows == [0]
