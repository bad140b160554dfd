"""Losslessness pin for the oracle by exact interval enumeration.

What the pages fix: verification is rejection sampling on the target/draft
probability ratio, and the tokens it emits are distributed exactly as the
target's own (umans.ai "DeepSeek V4 Pro DSpark: the model isn't ready, the
architecture is", section "Speculative decoding, briefly"; zhichai.net DSpark
topic, section "Why LLMs speak so slowly").  So, for every position i <= L,
given that positions 0..i-1 were emitted as accepted drafts, the token
emitted at position i must be distributed as the target's p_i, whatever the
prefix was.

The oracle's output is piecewise constant in each uniform it consumes.  For
every draft sequence x (weight prod_i q_i(x_i)) we evaluate the oracle once
per constant piece, at the piece's midpoint, and weight the result by the
piece's length.  The pieces come from p and q computed here with numpy from
the definition of a temperature softmax; if the oracle's breakpoints
differed, a piece would not be constant and the enumerated distribution would
miss the target.  The result is exact to rounding (1e-12).
"""
import itertools
from collections import defaultdict

import numpy as np
import pytest

import oracle


def softmax(z, T):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


def enumerate_outputs(zt, zd, L, T):
    """Exact distribution of the oracle's emitted token tuple."""
    K = zt.shape[0] - 1
    V = zt.shape[1]
    p = [softmax(zt[i], T) for i in range(K + 1)]
    q = None if zd is None else [softmax(zd[i], T) for i in range(K)]
    dist = defaultdict(float)

    def run(x, u_acc, j, u_res_j):
        ua = np.full(K + 1, 0.5)
        ua[:len(u_acc)] = u_acc
        ur = np.full(K + 1, 0.5)
        ur[j] = u_res_j
        xx = np.zeros(K, dtype=np.int32)
        xx[:len(x)] = x
        a, out, _ = oracle.verify_row_u(zt, zd, xx, L, T, ua, ur)
        return tuple(int(t) for t in out[:a + 1])

    def resample(x, u_acc, j, w, r):
        R = r.sum()
        C = np.cumsum(r) / R
        prev = 0.0
        for v in range(V):
            if r[v] > 0:
                dist[run(x, u_acc, j, 0.5 * (prev + C[v]))] += w * r[v] / R
            prev = C[v]

    def rec(x, i, u_acc, w):
        if i == L:
            resample(x, u_acc, L, w, p[L])
            return
        qi = 1.0 if q is None else q[i][x[i]]
        rho = min(1.0, p[i][x[i]] / qi)
        if rho > 0:
            rec(x, i + 1, u_acc + [0.5 * rho], w * rho)
        if rho < 1:
            sub = np.zeros(V)
            if q is None:
                sub[x[i]] = 1.0
            else:
                sub = q[i]
            resample(x, u_acc + [0.5 * (1.0 + rho)], i, w * (1.0 - rho),
                     np.maximum(0.0, p[i] - sub))

    if L == 0:
        rec((), 0, [], 1.0)
        return dist, p, q
    if q is None:
        # Greedy drafter: x is fixed; enumerate every fixed x separately.
        return None, p, q
    for x in itertools.product(range(V), repeat=L):
        w = float(np.prod([q[i][x[i]] for i in range(L)]))
        if w > 0:
            rec(x, 0, [], w)
    return dist, p, q


def check_lossless(dist, p, L, tol=1e-12):
    total = sum(dist.values())
    assert abs(total - 1.0) < tol
    V = p[0].size
    for i in range(L + 1):
        # group outputs that emitted at least i+1 tokens by their first i tokens
        by_prefix = defaultdict(lambda: np.zeros(V))
        for toks, pr in dist.items():
            if len(toks) >= i + 1:
                by_prefix[toks[:i]][toks[i]] += pr
        for prefix, mass in by_prefix.items():
            M = mass.sum()
            np.testing.assert_allclose(mass, M * p[i], rtol=0, atol=tol,
                                       err_msg=f"position {i} prefix {prefix}")


CASES = [(V, K) for V in (1, 2, 3, 5) for K in (1, 2, 3)] + [(8, 1), (8, 2)]


@pytest.mark.parametrize("V,K", CASES)
@pytest.mark.parametrize("T", [0.6, 1.0])
def test_sampled_drafter_is_lossless(V, K, T):
    rng = np.random.default_rng(1000 * V + 10 * K + int(T * 10))
    zt = rng.normal(0, 1.5, size=(K + 1, V))
    zd = zt[:K] + rng.normal(0, 1.0, size=(K, V))
    for L in range(K + 1):
        dist, p, q = enumerate_outputs(zt, zd, L, T)
        check_lossless(dist, p, L)
        # closed form: P(a >= i) = prod_{j<i} beta_j, beta_j = sum_v min(p_j, q_j)
        for i in range(L + 1):
            pa = sum(pr for toks, pr in dist.items() if len(toks) >= i + 1)
            beta = np.prod([np.minimum(p[j], q[j]).sum() for j in range(i)])
            assert abs(pa - beta) < 1e-12


@pytest.mark.parametrize("V,K", [(2, 2), (3, 3), (5, 2), (8, 1)])
def test_greedy_drafter_is_lossless_for_every_fixed_draft(V, K):
    """q_i one-hot at x_i: the emitted token at each position still follows p_i
    for any fixed draft sequence."""
    rng = np.random.default_rng(77 + V + K)
    zt = rng.normal(0, 1.5, size=(K + 1, V))
    T = 0.8
    p = [softmax(zt[i], T) for i in range(K + 1)]
    for L in range(K + 1):
        for x in itertools.product(range(V), repeat=L):
            dist = defaultdict(float)
            xx = np.zeros(K, dtype=np.int32)
            xx[:L] = x

            def run(u_acc, j, u):
                ua = np.full(K + 1, 0.5)
                ua[:len(u_acc)] = u_acc
                ur = np.full(K + 1, 0.5)
                ur[j] = u
                a, out, _ = oracle.verify_row_u(zt, None, xx, L, T, ua, ur)
                return tuple(int(t) for t in out[:a + 1])

            def resample(u_acc, j, w, r):
                C = np.cumsum(r) / r.sum()
                prev = 0.0
                for v in range(V):
                    if r[v] > 0:
                        dist[run(u_acc, j, 0.5 * (prev + C[v]))] += w * r[v] / r.sum()
                    prev = C[v]

            def rec(i, u_acc, w):
                if i == L:
                    resample(u_acc, L, w, p[L])
                    return
                rho = p[i][x[i]]
                rec(i + 1, u_acc + [0.5 * rho], w * rho)
                r = p[i].copy()
                r[x[i]] = 0.0
                if r.sum() > 0:
                    resample(u_acc + [0.5 * (1 + rho)], i, w * (1 - rho), r)

            rec(0, [], 1.0)
            check_lossless(dist, p, L)


def test_accept_breakpoint_is_min_one_ratio():
    """The accept decision flips exactly at u = min(1, p(x)/q(x))."""
    rng = np.random.default_rng(5)
    V, K = 6, 2
    for trial in range(40):
        zt = rng.normal(0, 2, size=(K + 1, V))
        zd = zt[:K] + rng.normal(0, 1.5, size=(K, V))
        T = [0.6, 1.0, 1.7][trial % 3]
        x = rng.integers(0, V, size=K).astype(np.int32)
        rho = min(1.0, softmax(zt[0], T)[x[0]] / softmax(zd[0], T)[x[0]])
        if not (1e-6 < rho < 1 - 1e-6):
            continue
        ur = np.full(K + 1, 0.5)
        a_lo, _, _ = oracle.verify_row_u(zt, zd, x, 1, T, [rho - 1e-9, 0.5, 0.5], ur)
        a_hi, _, _ = oracle.verify_row_u(zt, zd, x, 1, T, [rho + 1e-9, 0.5, 0.5], ur)
        assert a_lo == 1 and a_hi == 0


def test_residual_draw_is_inverse_cdf_in_token_order():
    """Reject at position 0; the correction token walks the residual CDF in
    token order with a strict '>' boundary."""
    zt = np.log(np.array([[0.1, 0.5, 0.4], [1 / 3, 1 / 3, 1 / 3]]))
    zd = np.log(np.array([[0.6, 0.2, 0.2]]))
    # residual max(0, p - q) = [0, 0.3, 0.2], R = 0.5 -> CDF breaks at 0.6, 1.0
    x = np.array([0], dtype=np.int32)        # ratio 0.1/0.6, so u=0.9 rejects
    for u, want in [(0.0, 1), (0.59, 1), (0.61, 2), (0.999, 2)]:
        a, out, diag = oracle.verify_row_u(zt, zd, x, 1, 1.0, [0.9, 0.5], [u, 0.5])
        assert a == 0 and out[0] == want, (u, out)
        assert abs(diag[4] - 0.5) < 1e-12
