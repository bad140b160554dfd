"""Helpers for GPU-vs-oracle parity: run both sides on the same seeded
inputs and compare row by row.

Every row is checked; none is excluded.  A row must either equal the
oracle's own result bit for bit, or be one of the outcomes the oracle lists
for decisions that lie inside the tie windows (``oracle.verify_window``):
an accept test with |u - min(1, ratio)| < 1e-5 may go either way, a final
draw may land on any token its target reaches within 1e-5 * R, and a
survival product within 1e-6 of tau may keep or drop its position.  The
outcome sets come from the oracle alone; the GPU result is only checked for
membership (``oracle.compare``).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import compare as ocompare
import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200.workloads import to_host_logits

ACCEPT_TIE = oracle.ACCEPT_WINDOW
CDF_TIE = oracle.CDF_WINDOW
SCHEDULE_TIE = oracle.SCHEDULE_WINDOW


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
    nt = oracle.default_threads()
    out, acc, diag, st = oracle.verify(zt_h, zd_h, tok, ln, tmp, seed, row_base=row_base,
                                       row_ids=rid, nthreads=nt)
    alt, _ = oracle.verify_window(zt_h, zd_h, tok, ln, tmp, seed, row_base=row_base,
                                  row_ids=rid, nthreads=nt)
    return dict(tokens=out, accept=acc, diag=diag, status=st, alt=alt, x=tok, lengths=ln)


def compare(g, o, rows=None):
    """Row-by-row check of a GPU result against the oracle result ``o`` (from
    :func:`oracle_verify`, same lengths on both sides).  Raises unless every
    row is bit-exact or one of the oracle's tie-window outcomes.  Returns the
    counts: rows, bit_exact, window_valid (rows that differ from the oracle's
    own result but lie inside a window), ties (rows with any window)."""
    gt = g["tokens"] if rows is None else g["tokens"][rows]
    ga = g["accept"] if rows is None else g["accept"][rows]
    alt = o["alt"]
    n = len(ga)
    alts = [[tuple(r) for r in alt[q] if r[0] >= 0] for q in range(n)]
    L = np.asarray(o["lengths"])
    t = ocompare.classify(np.arange(n) if rows is None else np.asarray(rows), o["x"],
                          o["tokens"], o["accept"], alt, alts, L, L, L, L, gt, ga)
    if t.invalid:
        raise AssertionError(f"{t.invalid} rows are neither bit-exact nor inside a tie window; "
                             f"first: {t.first_invalid}")
    ties = sum(1 for q in range(n) if len(alts[q]) > 1 or any(r[2] != r[3] for r in alts[q]))
    return dict(rows=n, bit_exact=t.bit_exact, window_valid=t.window_valid, ties=ties,
                tie_mismatches=t.window_valid)


def check_batch(batch, ln_gpu, g, seed, rows=None, row_base=0):
    """Complete check of a GPU verification of ``batch`` whose lengths came
    from ``sv_schedule`` (or are fixed): the oracle schedules on its own (rows
    whose survival product sits within the schedule window may take either
    length), then every row in ``rows`` (default all) must be bit-exact or a
    tie-window outcome.  Logits are copied to the host in row blocks."""
    tok = batch.tokens.cpu().numpy()
    tmp = batch.temperature.cpu().numpy()
    if batch.lengths is None:
        L0, lo, hi = ocompare.schedule_span(batch.conf.cpu().numpy(), batch.tau)
    else:
        L0 = batch.lengths.cpu().numpy()
        lo = hi = L0

    def fetch(idx):
        ix = torch.as_tensor(idx, device=batch.zt.device, dtype=torch.long)
        zd = None if batch.zd is None else to_host_logits(batch.zd.index_select(0, ix))
        return to_host_logits(batch.zt.index_select(0, ix)), zd

    t = ocompare.check_rows(fetch, tok, tmp, seed, L0, lo, hi, ln_gpu.cpu().numpy(),
                            g["tokens"], g["accept"], rows=rows, row_base=row_base)
    if t.invalid:
        raise AssertionError(f"{t.invalid} rows are neither bit-exact nor inside a tie window; "
                             f"first: {t.first_invalid}")
    return t.summary()


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
