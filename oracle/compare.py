"""Row-by-row comparison of a verification result with the oracle.

TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product.  It imports nothing from
the product; the result to check comes in as plain numpy arrays.

Every row is put in one of three classes:

* ``bit_exact``: accepted length and every output token equal the oracle's
  own result (and the verify length equals the oracle's schedule);
* ``window_valid``: not bit-exact, but the row is one of the outcomes the
  oracle lists for decisions inside the tie windows (``verify_window``): the
  verify length lies in the schedule window, the accepted length a is
  reachable, the first a tokens are the drafts, token a lies in the span
  [lo, hi] of that outcome's draw window, and the rest is -1;
* ``invalid``: anything else.  A correct implementation has none.

The outcome sets come from the oracle alone, on the oracle's own inputs
(its schedule, its uniforms); the result under test is only checked for
membership.  Rows whose schedule lies in a window are expanded over every
length the window allows.

The rule the windows follow: the emitted tokens must be distributed exactly
as the target's (umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready,
the architecture is", section "Speculative decoding, briefly"); a decision
within rounding of its threshold may go either way without changing that
distribution by more than the window's probability.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Optional

import numpy as np

from . import (ACCEPT_WINDOW, CDF_WINDOW, SCHEDULE_WINDOW, default_threads, schedule, verify,
               verify_window)


@dataclass
class Tally:
    rows: int = 0
    bit_exact: int = 0
    window_valid: int = 0
    invalid: int = 0
    accept_window_rows: int = 0     # rows whose accept tests reach more than one outcome
    cdf_window_rows: int = 0        # rows whose own draw window spans more than one token
    schedule_window_rows: int = 0   # rows whose verify length may take more than one value
    first_invalid: Optional[str] = None
    invalid_rows: list = field(default_factory=list)

    def add(self, other: "Tally") -> None:
        for k in ("rows", "bit_exact", "window_valid", "invalid", "accept_window_rows",
                  "cdf_window_rows", "schedule_window_rows"):
            setattr(self, k, getattr(self, k) + getattr(other, k))
        if self.first_invalid is None:
            self.first_invalid = other.first_invalid
        self.invalid_rows += other.invalid_rows

    def summary(self) -> dict:
        return {"rows": self.rows, "bit_exact": self.bit_exact,
                "window_valid": self.window_valid, "invalid": self.invalid,
                "in_window": {"accept": self.accept_window_rows, "cdf": self.cdf_window_rows,
                              "schedule": self.schedule_window_rows}}


def schedule_span(conf: np.ndarray, tau: float, w: float = SCHEDULE_WINDOW):
    """The oracle's verify lengths and the range each may take inside the
    schedule window: (L, L_lo, L_hi) with L_lo = #{i : S_i >= tau + w} and
    L_hi = #{i : S_i >= tau - w} (S is non-increasing along a row)."""
    L, S, _ = schedule(conf, tau)
    lo = (S >= tau + w).sum(axis=1).astype(np.int32)
    hi = (S >= tau - w).sum(axis=1).astype(np.int32)
    return L, lo, hi


def _row_ok(tok_row, a, x_row, K, alts):
    """Is (a, tokens) one of the listed outcomes?"""
    if a < 0:
        return False
    if not np.array_equal(tok_row[:a], x_row[:a]):
        return False
    if np.any(tok_row[a + 1:] != -1):
        return False
    y = int(tok_row[a])
    for (aa, _, lo, hi) in alts:
        if aa == a and lo <= y <= hi:
            return True
    return False


def check_rows(fetch: Callable, tokens: np.ndarray, temperature: np.ndarray, seed: int,
               lengths_oracle: np.ndarray, lengths_lo: np.ndarray, lengths_hi: np.ndarray,
               got_lengths: np.ndarray, got_tokens: np.ndarray, got_accept: np.ndarray,
               rows: Optional[np.ndarray] = None, row_base: int = 0, block: int = 64,
               nthreads: int = 0, w_acc: float = ACCEPT_WINDOW,
               w_cdf: float = CDF_WINDOW) -> Tally:
    """Classify every row in ``rows`` (default: all).

    fetch(idx) -> (zt [n, K+1, V], zd [n, K, V] or None) returns host logits
    (float32 or raw bf16 bits) of the batch rows idx; rows are fetched in
    blocks of ``block`` to bound host memory.  tokens [B, K] and temperature
    [B] are the batch inputs; lengths_* [B] come from :func:`schedule_span`
    (or all equal to fixed lengths); got_* are the result under test.
    The Philox row id of batch row b is row_base + b."""
    B = tokens.shape[0]
    K = tokens.shape[1]
    nthreads = nthreads or default_threads()
    idx_all = np.arange(B) if rows is None else np.asarray(rows)
    total = Tally()
    for s in range(0, len(idx_all), block):
        idx = idx_all[s:s + block]
        zt, zd = fetch(idx)
        tok = tokens[idx]
        tmp = temperature[idx]
        rid = idx.astype(np.int64) + row_base
        L0 = lengths_oracle[idx]
        o_tok, o_acc, _, _ = verify(zt, zd, tok, L0, tmp, seed, row_ids=rid, nthreads=nthreads)
        alt0, _ = verify_window(zt, zd, tok, L0, tmp, seed, w_acc=w_acc, w_cdf=w_cdf,
                                row_ids=rid, nthreads=nthreads)
        alts = [[tuple(r) for r in alt0[q] if r[0] >= 0] for q in range(len(idx))]
        # rows whose schedule may take other lengths: add those outcomes too
        span = np.flatnonzero(lengths_lo[idx] != lengths_hi[idx])
        for L in range(int(lengths_lo[idx].min(initial=0)), int(lengths_hi[idx].max(initial=0)) + 1):
            sel = [q for q in span if lengths_lo[idx[q]] <= L <= lengths_hi[idx[q]] and L != L0[q]]
            if not sel:
                continue
            sel = np.asarray(sel)
            altL, _ = verify_window(zt[sel], None if zd is None else zd[sel], tok[sel],
                                    np.full(len(sel), L, dtype=np.int32), tmp[sel], seed,
                                    w_acc=w_acc, w_cdf=w_cdf, row_ids=rid[sel],
                                    nthreads=nthreads)
            for k, q in enumerate(sel):
                alts[q] += [tuple(r) for r in altL[k] if r[0] >= 0]
        total.add(classify(idx, tok, o_tok, o_acc, alt0, alts, L0, lengths_lo[idx],
                           lengths_hi[idx], got_lengths[idx], got_tokens[idx],
                           got_accept[idx]))
    return total


def classify(row_ids, tokens, o_tok, o_acc, alt_own, alts, L0, L_lo, L_hi, got_lengths,
             got_tokens, got_accept) -> Tally:
    """Classify rows given the oracle's own result (o_tok, o_acc at lengths
    L0), its outcome set alt_own [n, K+1, 4] at L0, and the full outcome set
    alts (a list per row of (a, y, lo, hi), every allowed length included).
    row_ids only label the rows in the report."""
    t = Tally()
    K = tokens.shape[1]
    for q, b in enumerate(row_ids):
        t.rows += 1
        own = [r for r in alt_own[q] if r[0] >= 0]
        if len(own) > 1:
            t.accept_window_rows += 1
        if own and any(r[2] != r[3] for r in own):
            t.cdf_window_rows += 1
        if L_lo[q] != L_hi[q]:
            t.schedule_window_rows += 1
        gl, ga, gt = int(got_lengths[q]), int(got_accept[q]), got_tokens[q]
        if gl == L0[q] and ga == o_acc[q] and np.array_equal(gt, o_tok[q]):
            t.bit_exact += 1
            continue
        ok = (L_lo[q] <= gl <= L_hi[q]) and ga <= gl and _row_ok(gt, ga, tokens[q], K, alts[q])
        if ok:
            t.window_valid += 1
        else:
            t.invalid += 1
            t.invalid_rows.append(int(b))
            if t.first_invalid is None:
                t.first_invalid = (f"row {int(b)}: got L={gl} a={ga} tokens={gt.tolist()}; "
                                   f"oracle L={int(L0[q])} (window {int(L_lo[q])}.."
                                   f"{int(L_hi[q])}) a={int(o_acc[q])} "
                                   f"tokens={o_tok[q].tolist()} outcomes={alts[q]}")
    return t
