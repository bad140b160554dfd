"""Distribution tests on GPU draws: the emitted tokens are distributed as
the target's (chi-square over 10^6 draws, V <= 8), and the mean accepted
length at a large vocabulary matches the closed form
E[a] = sum_{i=1..L} prod_{j<i} beta_j, beta_j = sum_v min(p_j, q_j)."""
import math

import numpy as np
import pytest
import torch
from scipy import stats as sst

from speculative_decoding_verification_93_b200 import workloads
from _parity import gpu_verify

pytestmark = pytest.mark.gpu


def softmax(z, T):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


def identical_rows(V, K, T, B, seed, dtype=torch.float32, noise=1.2, std=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    zt1 = (torch.randn(1, K + 1, V, generator=g, device="cuda") * std).to(dtype)
    zd1 = (zt1[:, :K].float() + noise * torch.randn(1, K, V, generator=g, device="cuda")).to(dtype)
    zt = zt1.expand(B, K + 1, V).contiguous()
    zd = zd1.expand(B, K, V).contiguous()
    temp = torch.full((B,), T, device="cuda")
    x = workloads.gumbel_tokens(zd, temp, g, rows_per_block=B)
    return zt, zd, x, temp


@pytest.mark.parametrize("V,T,dtype", [(5, 1.0, torch.float32), (8, 0.6, torch.bfloat16),
                                       (3, 1.0, torch.bfloat16)])
def test_emitted_tokens_follow_target_chi2(V, T, dtype):
    K, B, nseeds = 2, 10_000, 100
    zt, zd, _, temp = identical_rows(V, K, T, B, seed=V)
    L = torch.full((B,), K, dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(1234)
    counts = [np.zeros(V) for _ in range(K + 1)]
    for s in range(nseeds):
        x = workloads.gumbel_tokens(zd, temp, gen, rows_per_block=B)   # fresh drafts
        g = gpu_verify(zt, zd, x, L, temp, seed=s)
        for i in range(K + 1):
            sel = g["accept"] >= i
            counts[i] += np.bincount(g["tokens"][sel, i], minlength=V)
    ztn = zt[0].float().cpu().numpy()
    for i in range(K + 1):
        p = softmax(ztn[i], T)
        n = counts[i].sum()
        chi2 = ((counts[i] - n * p) ** 2 / (n * p)).sum()
        pv = sst.chi2.sf(chi2, V - 1)
        assert pv > 1e-3, (i, counts[i], n * p, pv)
    assert counts[0].sum() == B * nseeds


@pytest.mark.parametrize("V,K,T", [(129280, 4, 1.0), (32000, 6, 0.6)])
def test_mean_accept_length_closed_form(V, K, T):
    B = 4096
    zt, zd, x, temp = identical_rows(V, K, T, B, seed=3, dtype=torch.bfloat16, noise=0.8,
                                     std=3.0)
    L = torch.full((B,), K, dtype=torch.int32, device="cuda")
    g = gpu_verify(zt, zd, x, L, temp, seed=77)
    a = g["accept"].astype(np.float64)
    ztn = zt[0].float().cpu().numpy()
    zdn = zd[0].float().cpu().numpy()
    beta = [np.minimum(softmax(ztn[i], T), softmax(zdn[i], T)).sum() for i in range(K)]
    Ea = sum(np.prod(beta[:i]) for i in range(1, K + 1))
    se = a.std(ddof=1) / math.sqrt(B)
    assert abs(a.mean() - Ea) < 4 * se, (a.mean(), Ea, se)
