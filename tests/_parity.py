"""Helpers for GPU-vs-oracle parity: run both sides on the same seeded
inputs and compare element by element.

Tie windows (decisions that floating point may legitimately flip between the
fp32 kernels and the fp64 oracle) are taken from the oracle's own
diagnostics, never from the GPU: a row is excluded when one of its tested
positions has |u - min(1, ratio)| < 1e-5, when its final draw lies within
1e-5 * R of a CDF boundary, or when a survival product lies within 1e-6 of
tau.  Excluded rows are counted and returned; everything else must match bit
for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200.workloads import to_host_logits

ACCEPT_TIE = 1e-5
CDF_TIE = 1e-5
SCHEDULE_TIE = 1e-6


def gpu_verify(zt, zd, tokens, lengths, temperature, seed, row_base=0, debug=False,
               workspace=None):
    B, K1, V = zt.shape
    K = K1 - 1
    dev = zt.device
    dt = sv.SV_BF16 if zt.dtype == torch.bfloat16 else sv.SV_F32
    if workspace is None:
        workspace = torch.empty(sv.sv_verify_workspace_bytes(B, K, V, dt), dtype=torch.uint8,
                                device=dev)
    out_tok = torch.full((B, K1), -7, dtype=torch.int32, device=dev)
    out_acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stats = None
    if debug:
        stats = torch.full((B, 2 * K + 1, 2), float("nan"), dtype=torch.float32, device=dev)
        sv.sv_verify_debug(zt, zd, tokens, lengths, temperature, seed, out_tok, out_acc,
                           workspace, stats, status=status, row_base=row_base)
    else:
        sv.sv_verify(zt, zd, tokens, lengths, temperature, seed, out_tok, out_acc, workspace,
                     status=status, row_base=row_base)
    torch.cuda.synchronize()
    return dict(tokens=out_tok.cpu().numpy(), accept=out_acc.cpu().numpy(),
                status=int(status.item()),
                stats=None if stats is None else stats.cpu().numpy())


def gpu_schedule(conf, tau):
    B, K = conf.shape
    ln = torch.full((B,), -7, dtype=torch.int32, device=conf.device)
    sv.sv_schedule(conf, tau, ln)
    torch.cuda.synchronize()
    return ln


def oracle_verify(zt, zd, tokens, lengths_np, temperature, seed, rows=None, row_base=0):
    """Oracle on host copies; `rows` selects a subset (Philox keyed by the
    global row id)."""
    if rows is not None:
        idx = torch.as_tensor(rows, device=zt.device, dtype=torch.long)
        zt_h = to_host_logits(zt.index_select(0, idx))
        zd_h = None if zd is None else to_host_logits(zd.index_select(0, idx))
        tok = tokens.index_select(0, idx).cpu().numpy()
        tmp = temperature.index_select(0, idx).cpu().numpy()
        ln = np.asarray(lengths_np)[np.asarray(rows)]
        rid = np.asarray(rows, dtype=np.int64) + row_base
    else:
        zt_h = to_host_logits(zt)
        zd_h = None if zd is None else to_host_logits(zd)
        tok = tokens.cpu().numpy()
        tmp = temperature.cpu().numpy()
        ln = np.asarray(lengths_np)
        rid = None
    out, acc, diag, st = oracle.verify(zt_h, zd_h, tok, ln, tmp, seed, row_base=row_base,
                                       row_ids=rid, nthreads=oracle.default_threads())
    return dict(tokens=out, accept=acc, diag=diag, status=st)


def compare(g, o, rows=None, extra_excluded=None):
    """Element-by-element comparison; returns counts.  Raises on a mismatch
    outside the tie windows."""
    gt = g["tokens"] if rows is None else g["tokens"][rows]
    ga = g["accept"] if rows is None else g["accept"][rows]
    diag = o["diag"]
    tie = np.zeros(len(ga), dtype=bool)
    with np.errstate(invalid="ignore"):
        tie |= diag[:, 0] < ACCEPT_TIE
        tie |= diag[:, 1] < CDF_TIE
    if extra_excluded is not None:
        tie |= extra_excluded
    same = (ga == o["accept"]) & np.all(gt == o["tokens"], axis=1)
    bad = ~same & ~tie
    if bad.any():
        r = int(np.flatnonzero(bad)[0])
        raise AssertionError(
            f"{int(bad.sum())} rows differ outside the tie windows; first row {r}: "
            f"gpu a={ga[r]} tokens={gt[r].tolist()} oracle a={o['accept'][r]} "
            f"tokens={o['tokens'][r].tolist()} diag={diag[r].tolist()}")
    return dict(rows=len(ga), ties=int(tie.sum()), tie_mismatches=int((~same & tie).sum()))


def check_structure(g, tokens_np, lengths_np):
    """Invariants every output row must satisfy: 0 <= a <= L, the first a
    tokens are the drafts, exactly a+1 tokens, then -1."""
    B, K1 = g["tokens"].shape
    for b in range(B):
        a = g["accept"][b]
        if a < 0:
            assert np.all(g["tokens"][b] == -1)
            continue
        assert 0 <= a <= lengths_np[b]
        assert np.array_equal(g["tokens"][b, :a], tokens_np[b, :a])
        assert g["tokens"][b, a] >= 0
        assert np.all(g["tokens"][b, a + 1:] == -1)
