"""Vocabulary-parallel verification over a process group (one process per GPU).

Each rank holds a contiguous slice of the vocabulary of both models' logits,
as a serving engine whose output heads are split by vocabulary produces them
(zhichai.net DSpark topic, "From paper to running service in two weeks";
techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier", Ch. 7
"Deployment with vLLM").  One step is three entry points of ``libsv.so``
(four kernel launches: sv_vp_decide issues two) with three collectives
between them (``include/sv.h``, sv_vp_*):

    sv_vp_stats -> all-gather (rank order) -> sv_vp_decide
                -> all-gather (rank order) -> sv_vp_draw -> all-reduce(max)

The collectives move B * (2K+1) * C * 16 bytes, B * 8 bytes and
B * (K+1) * 4 bytes per rank; the logits never leave their GPU.  With one
rank the collectives are skipped.  Every step of the method runs in the
library's kernels; this module owns the buffers and issues the collectives.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _binding as _b
from .sharding import shard_rows


def shard_vocab(V: int, world: int, rank: int) -> Tuple[int, int]:
    """Slice [v0, v1) of rank `rank`: contiguous, in rank order, sizes that
    differ by at most one token (so no slice exceeds ceil(V / world))."""
    if V < world:
        raise ValueError("need at least one token per rank")
    return shard_rows(V, world, rank)


def _group_size_rank(group) -> Tuple[int, int]:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def gather_in_rank_order(local: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """out = concatenation of every rank's `local` along dim 0, rank order."""
    world, _ = _group_size_rank(group)
    if world == 1:
        if out.data_ptr() != local.data_ptr():
            out.copy_(local)
        return out
    import torch.distributed as dist
    dist.all_gather_into_tensor(out, local, group=group)
    return out


def reduce_tokens(out_tokens: torch.Tensor, group=None) -> torch.Tensor:
    """Element-wise max over the ranks: every rank writes the same accepted
    prefix and -1 at the drawn position except the rank that drew it."""
    world, _ = _group_size_rank(group)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(out_tokens, op=dist.ReduceOp.MAX, group=group)
    return out_tokens


class VocabParallelVerifier:
    """Buffers and collectives of vocabulary-parallel verification for a
    fixed (B, K, V, dtype) on this rank of `group`."""

    def __init__(self, B: int, K: int, V: int, dtype: torch.dtype, device, group=None,
                 with_draft: bool = True):
        self.group = group
        self.world, self.rank = _group_size_rank(group)
        self.B, self.K, self.V = B, K, V
        self.v0, v1 = shard_vocab(V, self.world, self.rank)
        self.Vs = v1 - self.v0
        self.dtype = dtype
        self.device = torch.device(device)
        codes = {torch.float32: _b.SV_F32, torch.bfloat16: _b.SV_BF16}
        if dtype not in codes:
            raise TypeError(f"logits must be float32 or bfloat16, got {dtype}")
        # Sizes depend on the shape only; the pointers are placeholders.
        desc = _b.sv_vp_slice(16, 16 if with_draft else None, codes[dtype], B, K, V, self.v0,
                              self.Vs, self.world, self.rank)
        n_stats = _b.sv_vp_stats_bytes(desc)
        n_ws = _b.sv_vp_workspace_bytes(desc)
        if n_stats == 0 or n_ws == 0:
            raise ValueError("unsupported vocabulary-parallel shape")
        self.stats_local = torch.empty(n_stats, dtype=torch.uint8, device=self.device)
        self.stats_all = (self.stats_local if self.world == 1 else
                          torch.empty(n_stats * self.world, dtype=torch.uint8, device=self.device))
        self.mass_local = torch.empty(B, 2, dtype=torch.float32, device=self.device)
        self.mass_all = (self.mass_local if self.world == 1 else
                         torch.empty(self.world * B, 2, dtype=torch.float32, device=self.device))
        self.workspace = torch.empty(n_ws, dtype=torch.uint8, device=self.device)

    def slice_of(self, target_logits: torch.Tensor,
                 draft_logits: Optional[torch.Tensor]) -> _b.sv_vp_slice:
        if target_logits.shape[-1] != self.Vs:
            raise ValueError(f"this rank holds {self.Vs} tokens, logits have "
                             f"{target_logits.shape[-1]}")
        return _b.vp_slice(target_logits, draft_logits, self.V, self.v0, self.world, self.rank)

    def step(self, target_logits, draft_logits, draft_tokens, lengths, temperature, seed: int,
             out_tokens, out_accept_len, status=None, row_base: int = 0, norm_out=None):
        """One verification step of this rank's slice; on return (stream
        order) every rank holds the full out_tokens and out_accept_len."""
        d = self.slice_of(target_logits, draft_logits)
        _b.sv_vp_stats(d, draft_tokens, lengths, temperature, self.stats_local)
        gather_in_rank_order(self.stats_local, self.stats_all, self.group)
        _b.sv_vp_decide(d, self.stats_all, draft_tokens, lengths, temperature, seed, out_tokens,
                        out_accept_len, self.mass_local, self.workspace, status=status,
                        norm_out=norm_out, row_base=row_base)
        gather_in_rank_order(self.mass_local, self.mass_all, self.group)
        _b.sv_vp_draw(d, self.mass_all, out_tokens, self.workspace, status=status)
        reduce_tokens(out_tokens, self.group)
        return out_tokens, out_accept_len
