"""Seeded synthetic workloads for verification (inputs only).

This module makes the inputs that both the CUDA path and the CPU oracle
consume.  It holds none of the verification arithmetic: no softmax
statistics, no acceptance test and no inverse-CDF draw.  Draft tokens are
drawn from the draft distribution with the Gumbel-max trick, which stands in
for the drafter's own sampling and is unrelated to the verifier's
inverse-CDF draw.

The workloads mirror the verification batches the pages describe: a drafter
proposes K tokens per request, the target scores K+1 positions in one pass
(umans.ai "DeepSeek V4 Pro DSpark: the model isn't ready, the architecture
is", section "Speculative decoding, briefly"), the vocabulary is the ~128K
DeepSeek tokenizer (V = 129280), and the drafter's per-position survival
confidences feed the verify-length schedule (same page, "What DSpark adds",
item "2. Verify smarter").  Parallel drafters lose acceptance down the block
("suffix decay", same page, item "1. Draft better"), which the growing
per-position draft noise of ``c4`` imitates.  The logits are synthetic
Gaussians: no trained weights or traffic are used.

Named workloads (B rows, K drafts, V vocabulary):

  c0  B=4,    K=4,  V=1000,   fp32  zt~N(0,3^2); zd = zt + N(0,1); T=1; L=4
  c1  B=64,   K=4,  V=129280, bf16  zt~N(0,3^2), one token per (row,pos)
                                    boosted by +8; zd = zt + N(0,s_b^2),
                                    s_b~U[0.5,2] per row; T=1; L=4
  c2  B=256,  K=8,  V=129280, bf16  logits as c1; T per row from
                                    {0, 0.6, 1.0}; conf~Beta(8,2), tau=0.3
  c3  B=1024, K=2,  V=129280, bf16  zt~N(0,2^2); zd = zt + N(0,0.7^2);
                                    T=0.8; L=2
  c4  B=512,  K=16, V=129280, fp32  zt~N(0,3^2); zd = zt + N(0,s_i^2),
                                    s_i = 0.3 + 2.7 i/15; T=1;
                                    conf~Beta(6,3), tau in {0.1,0.3,0.6}

Draft tokens: x_i ~ softmax(zd_i / T_b) (Gumbel-max), or argmax zd_i when
T_b = 0.  Data seed = workload index; verification seed 0.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

V_DEEPSEEK = 129280


@dataclass
class Spec:
    name: str
    B: int
    K: int
    V: int
    dtype: torch.dtype
    target_std: float
    boost: float                       # added to one random token per (row, pos); 0 = none
    draft_noise: str                   # "const", "per_row", "per_pos"
    noise_a: float
    noise_b: float
    temps: tuple                       # per-row temperature choices
    fixed_length: Optional[int]        # None: lengths come from the schedule
    beta: Optional[tuple] = None       # confidence Beta(a, b)
    taus: tuple = ()
    data_seed: int = 0
    verify_seed: int = 0


SPECS = {
    "c0": Spec("c0", 4, 4, 1000, torch.float32, 3.0, 0.0, "const", 1.0, 1.0, (1.0,), 4,
               data_seed=0),
    "c1": Spec("c1", 64, 4, V_DEEPSEEK, torch.bfloat16, 3.0, 8.0, "per_row", 0.5, 2.0, (1.0,), 4,
               data_seed=1),
    "c2": Spec("c2", 256, 8, V_DEEPSEEK, torch.bfloat16, 3.0, 8.0, "per_row", 0.5, 2.0,
               (0.0, 0.6, 1.0), None, beta=(8.0, 2.0), taus=(0.3,), data_seed=2),
    "c3": Spec("c3", 1024, 2, V_DEEPSEEK, torch.bfloat16, 2.0, 0.0, "const", 0.7, 0.7, (0.8,), 2,
               data_seed=3),
    "c4": Spec("c4", 512, 16, V_DEEPSEEK, torch.float32, 3.0, 0.0, "per_pos", 0.3, 3.0, (1.0,),
               None, beta=(6.0, 3.0), taus=(0.1, 0.3, 0.6), data_seed=4),
}


@dataclass
class Batch:
    """One verification batch.  Tensors live on ``device``."""
    spec: Spec
    zt: torch.Tensor            # [B, K+1, V]
    zd: torch.Tensor            # [B, K, V]
    tokens: torch.Tensor        # [B, K] int32
    temperature: torch.Tensor   # [B] float32
    conf: torch.Tensor          # [B, K] float32
    tau: float
    lengths: Optional[torch.Tensor]   # [B] int32, or None (take from the schedule)
    extra: dict = field(default_factory=dict)


def _row_sigmas(spec: Spec, rng: np.random.Generator, B: int, K: int) -> np.ndarray:
    """Standard deviation of the draft noise, shape [B, K]."""
    if spec.draft_noise == "const":
        return np.full((B, K), spec.noise_a)
    if spec.draft_noise == "per_row":
        return np.repeat(rng.uniform(spec.noise_a, spec.noise_b, size=(B, 1)), K, axis=1)
    if spec.draft_noise == "per_pos":
        i = np.arange(K, dtype=np.float64)
        s = spec.noise_a + (spec.noise_b - spec.noise_a) * i / max(K - 1, 1)
        return np.repeat(s[None, :], B, axis=0)
    raise ValueError(spec.draft_noise)


def gumbel_tokens(zd: torch.Tensor, temperature: torch.Tensor, gen: torch.Generator,
                  rows_per_block: int = 16) -> torch.Tensor:
    """Draw x_i ~ softmax(zd_i / T_b) by Gumbel-max (argmax when T_b == 0).

    Stands in for the drafter's own sampling; processed in row blocks to keep
    the temporary at a few hundred MB."""
    B, K, V = zd.shape
    out = torch.empty(B, K, dtype=torch.int32, device=zd.device)
    for r0 in range(0, B, rows_per_block):
        r1 = min(B, r0 + rows_per_block)
        z = zd[r0:r1].float()
        T = temperature[r0:r1].float().view(-1, 1, 1)
        u = torch.rand(z.shape, generator=gen, device=z.device, dtype=torch.float32)
        u = u.clamp_(min=1e-12, max=1.0 - 1e-7)
        g = -torch.log(-torch.log(u))
        greedy = (T == 0)
        score = torch.where(greedy, z, z / torch.where(greedy, torch.ones_like(T), T) + g)
        out[r0:r1] = score.argmax(dim=-1).to(torch.int32)
        del z, u, g, score
    return out


def make_batch(name: str, device="cpu", B: Optional[int] = None, V: Optional[int] = None,
               tau: Optional[float] = None, data_seed: Optional[int] = None,
               rows_per_block: int = 16) -> Batch:
    """Generate workload ``name`` (optionally with B or V overridden for
    smaller parity cases)."""
    spec = SPECS[name]
    B = spec.B if B is None else B
    V = spec.V if V is None else V
    K = spec.K
    seed = spec.data_seed if data_seed is None else data_seed
    rng = np.random.default_rng(seed)
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)

    temps = rng.choice(np.asarray(spec.temps, dtype=np.float32), size=B).astype(np.float32)
    sig = _row_sigmas(spec, rng, B, K).astype(np.float32)
    boost_idx = rng.integers(0, V, size=(B, K + 1))
    if spec.beta is not None:
        conf = rng.beta(spec.beta[0], spec.beta[1], size=(B, K)).astype(np.float32)
    else:
        conf = np.ones((B, K), dtype=np.float32)
    tau_v = (spec.taus[0] if spec.taus else 0.0) if tau is None else tau

    zt = torch.empty(B, K + 1, V, dtype=spec.dtype, device=dev)
    zd = torch.empty(B, K, V, dtype=spec.dtype, device=dev)
    sig_t = torch.from_numpy(sig).to(dev)
    bidx = torch.from_numpy(boost_idx).to(dev)
    for r0 in range(0, B, rows_per_block):
        r1 = min(B, r0 + rows_per_block)
        t = torch.randn(r1 - r0, K + 1, V, generator=gen, device=dev) * spec.target_std
        if spec.boost:
            t.scatter_add_(2, bidx[r0:r1].unsqueeze(-1),
                           torch.full((r1 - r0, K + 1, 1), spec.boost, device=dev))
        t = t.to(spec.dtype)
        zt[r0:r1] = t
        n = torch.randn(r1 - r0, K, V, generator=gen, device=dev) * sig_t[r0:r1].unsqueeze(-1)
        zd[r0:r1] = (t[:, :K].float() + n).to(spec.dtype)
        del t, n
    temperature = torch.from_numpy(temps).to(dev)
    tokens = gumbel_tokens(zd, temperature, gen, rows_per_block)
    lengths = None
    if spec.fixed_length is not None:
        lengths = torch.full((B,), spec.fixed_length, dtype=torch.int32, device=dev)
    return Batch(spec=spec, zt=zt, zd=zd, tokens=tokens, temperature=temperature,
                 conf=torch.from_numpy(conf).to(dev), tau=float(tau_v), lengths=lengths)


def random_small(B: int, K: int, V: int, dtype=torch.float32, seed: int = 0,
                 target_std: float = 3.0, noise: float = 1.0, temps=(1.0,),
                 lengths=None, device="cpu") -> Batch:
    """Small adversarial/parity batch with explicit sizes."""
    rng = np.random.default_rng(seed)
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    t = (torch.randn(B, K + 1, V, generator=gen, device=dev) * target_std)
    zt = t.to(dtype)
    zd = (zt[:, :K].float() + noise * torch.randn(B, K, V, generator=gen, device=dev)).to(dtype)
    temperature = torch.from_numpy(
        rng.choice(np.asarray(temps, dtype=np.float32), size=B).astype(np.float32)).to(dev)
    tokens = gumbel_tokens(zd, temperature, gen)
    if lengths is None:
        ln = torch.from_numpy(rng.integers(0, K + 1, size=B).astype(np.int32)).to(dev)
    elif np.isscalar(lengths):
        ln = torch.full((B,), int(lengths), dtype=torch.int32, device=dev)
    else:
        ln = torch.as_tensor(np.asarray(lengths, dtype=np.int32), device=dev)
    conf = torch.from_numpy(rng.beta(8.0, 2.0, size=(B, K)).astype(np.float32)).to(dev)
    return Batch(spec=Spec("small", B, K, V, dtype, target_std, 0.0, "const", noise, noise,
                           tuple(temps), None),
                 zt=zt, zd=zd, tokens=tokens, temperature=temperature, conf=conf, tau=0.3,
                 lengths=ln)


def to_host_logits(t: torch.Tensor) -> np.ndarray:
    """Logits as a numpy array for the oracle: float32 as is, bf16 as its raw
    16-bit patterns (uint16)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def sts_heldout(N: int, K: int, seed: int = 0, kappa=(1.3, 2.2), mu: float = 1.8,
                sigma: float = 1.0):
    """Synthetic held-out blocks for the confidence head's calibration: a
    true survival logit l* ~ N(mu, sigma^2) per (block, position); survival
    drawn left to right from sigmoid(l*) until the first failure (the
    accepted length a); the head reports l = kappa_i * l*, overconfident by
    a factor kappa_i spread evenly over `kappa` along the block.  Returns
    (logits [N, K] float32, accept [N] int32), numpy."""
    rng = np.random.default_rng(seed)
    lstar = rng.normal(mu, sigma, size=(N, K))
    kap = np.linspace(kappa[0], kappa[1], K)
    logits = (lstar * kap).astype(np.float32)
    survive = rng.random((N, K)) < 1.0 / (1.0 + np.exp(-lstar))
    accept = np.where(survive.all(axis=1), K, np.argmin(survive, axis=1)).astype(np.int32)
    return logits, accept
