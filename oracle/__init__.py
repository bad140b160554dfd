"""fp64 CPU oracle for confidence-scheduled speculative verification.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never loads it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64); this module only
marshals numpy arrays through ctypes.  Every function follows the pages cited
in ``oracle.c``'s header:

* speculative rejection sampling: umans.ai "DeepSeek V4 Pro DSpark: the model
  isn't ready, the architecture is", section "Speculative decoding, briefly";
  zhichai.net DSpark topic, section "Why LLMs speak so slowly";
* prefix survival and the load threshold: same umans.ai page, section "What
  DSpark adds", item "2. Verify smarter"; aiweekly.co alert; techvisionai
  "DeepSeek-V4: Breaking the Efficiency Barrier", Ch. 7
  "Confidence-Scheduled Verification";
* Philox4x32-10: Salmon et al., SC'11.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, F64 = 0, 1, 2
NDIAG = 5

# Tie windows for comparing an fp32 implementation with this fp64 oracle.
# An accept test with |u - min(1, ratio)| below ACCEPT_WINDOW may go either
# way.  A final draw may land on any token its target reaches when moved by
# up to CDF_WINDOW * R (the same bound, read onto the inverse CDF).  A
# survival product with |S_i - tau| below SCHEDULE_WINDOW may keep or drop
# position i (fp32 products against fp64).
ACCEPT_WINDOW = 1e-5
CDF_WINDOW = 1e-5
SCHEDULE_WINDOW = 1e-6

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, i64, u64, dbl = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                  ctypes.c_uint64, ctypes.c_double)
        L.oracle_philox4x32_10.argtypes = [vp, vp, vp]
        L.oracle_philox4x32_10.restype = None
        L.oracle_uniform.argtypes = [u64, u64, ctypes.c_uint32, ctypes.c_uint32]
        L.oracle_uniform.restype = dbl
        L.oracle_uniform_batch.argtypes = [u64, vp, vp, vp, i64, vp]
        L.oracle_uniform_batch.restype = None
        L.oracle_verify_row_u.argtypes = [vp, vp, i32, i32, vp, i32, dbl, vp, vp, vp, vp]
        L.oracle_verify_row_u.restype = i32
        L.oracle_verify.argtypes = [vp, vp, i32, i64, i32, i32, vp, vp, vp, u64, i64, vp,
                                    vp, vp, vp, i32]
        L.oracle_verify.restype = i32
        L.oracle_verify_window.argtypes = [vp, vp, i32, i64, i32, i32, vp, vp, vp, u64, i64,
                                           vp, dbl, dbl, vp, i32]
        L.oracle_verify_window.restype = i32
        L.oracle_verify_window_row_u.argtypes = [vp, vp, i32, i32, vp, i32, dbl, vp, vp, dbl,
                                                 dbl, vp]
        L.oracle_verify_window_row_u.restype = i32
        L.oracle_stats_batch.argtypes = [vp, i32, i64, i32, vp, vp, vp, vp, i32]
        L.oracle_stats_batch.restype = None
        L.oracle_schedule.argtypes = [vp, i64, i32, dbl, vp, vp]
        L.oracle_schedule.restype = dbl
        L.oracle_schedule_admit.argtypes = [vp, i32, i32, vp, i32, vp, vp, vp]
        L.oracle_schedule_admit.restype = i32
        L.oracle_ndiag.restype = i32
        L.oracle_sts_fit.argtypes = [vp, vp, i32, i32, dbl, dbl, vp, vp]
        L.oracle_sts_fit.restype = ctypes.c_long
        assert L.oracle_ndiag() == NDIAG
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:  # raw bf16 bits
        return BF16
    raise TypeError(f"logits must be float32 or raw bf16 bits (uint16), got {a.dtype}")


def philox4x32_10(ctr, key) -> np.ndarray:
    """Raw Philox4x32-10 block for one counter (4 x u32) and key (2 x u32)."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().oracle_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def uniform(seed: int, row: int, pos: int, draw: int) -> float:
    """u(seed, row, pos, draw) = (word0 >> 8) * 2^-24 of Philox4x32-10 with
    key (seed_lo, seed_hi) and counter (row_lo, pos, draw, row_hi)."""
    return lib().oracle_uniform(seed, row, pos, draw)


def uniform_batch(seed: int, row, pos, draw) -> np.ndarray:
    """Vectorised :func:`uniform` over equal-length arrays."""
    r = np.ascontiguousarray(row, dtype=np.uint64)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.uint32), r.shape))
    d = np.ascontiguousarray(np.broadcast_to(np.asarray(draw, dtype=np.uint32), r.shape))
    out = np.zeros(r.shape, dtype=np.float64)
    lib().oracle_uniform_batch(ctypes.c_uint64(seed & (2**64 - 1)), _p(r), _p(p), _p(d),
                               r.size, _p(out))
    return out


def verify_row_u(zt, zd, x, L, T, u_acc, u_res):
    """One row, fp64 logits, injected uniforms.

    zt [K+1, V], zd [K, V] or None (greedy drafter), x [K], u_acc [K+1],
    u_res [K+1].  Returns (a, out_tokens [K+1], diag [NDIAG])."""
    zt = np.ascontiguousarray(zt, dtype=np.float64)
    K1, V = zt.shape
    K = K1 - 1
    zd_a = None if zd is None else np.ascontiguousarray(zd, dtype=np.float64)
    if zd_a is not None:
        assert zd_a.shape == (K, V)
    x = np.ascontiguousarray(x, dtype=np.int32).reshape(K)
    ua = np.ascontiguousarray(u_acc, dtype=np.float64).reshape(-1)
    ur = np.ascontiguousarray(u_res, dtype=np.float64).reshape(-1)
    assert ua.size >= K + 1 and ur.size >= K + 1
    out = np.zeros(K + 1, dtype=np.int32)
    diag = np.zeros(NDIAG, dtype=np.float64)
    a = lib().oracle_verify_row_u(_p(zt), _p(zd_a), K, V, _p(x), int(L), float(T),
                                  _p(ua), _p(ur), _p(out), _p(diag))
    if a < 0:
        raise ValueError("oracle_verify_row_u: bad arguments")
    return a, out, diag


def verify(zt, zd, tokens, lengths, temperature, seed, row_base=0, row_ids=None,
           nthreads=0):
    """Batch verification with Philox-keyed uniforms.

    zt [B, K+1, V] and zd [B, K, V] (or None) as float32 or raw bf16 bits
    (uint16).  Returns (out_tokens [B, K+1], out_accept [B], diag [B, NDIAG],
    status bits)."""
    zt = np.ascontiguousarray(zt)
    B, K1, V = zt.shape
    K = K1 - 1
    dt = _dtype_code(zt)
    if zd is not None:
        zd = np.ascontiguousarray(zd)
        assert zd.shape == (B, K, V) and zd.dtype == zt.dtype
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, K)
    ln = np.ascontiguousarray(lengths, dtype=np.int32).reshape(B)
    tp = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    rid = None if row_ids is None else np.ascontiguousarray(row_ids, dtype=np.int64).reshape(B)
    out = np.zeros((B, K + 1), dtype=np.int32)
    acc = np.zeros(B, dtype=np.int32)
    diag = np.zeros((B, NDIAG), dtype=np.float64)
    st = lib().oracle_verify(_p(zt), _p(zd), dt, B, K, V, _p(tok), _p(ln), _p(tp),
                             ctypes.c_uint64(seed & (2**64 - 1)), int(row_base), _p(rid),
                             _p(out), _p(acc), _p(diag), int(nthreads))
    return out, acc, diag, st


def verify_window(zt, zd, tokens, lengths, temperature, seed, w_acc=ACCEPT_WINDOW,
                  w_cdf=CDF_WINDOW, row_base=0, row_ids=None, nthreads=0):
    """Every outcome the rule allows when each accept test may flip within
    w_acc of its threshold and each final draw may move within w_cdf * R of
    its target (see oracle_verify_window in oracle.c).

    Same inputs as :func:`verify`.  Returns (alt [B, K+1, 4] int32 of
    (a, y, lo, hi) per reachable accepted length a, in increasing a, padded
    with -1; status bits)."""
    zt = np.ascontiguousarray(zt)
    B, K1, V = zt.shape
    K = K1 - 1
    dt = _dtype_code(zt)
    if zd is not None:
        zd = np.ascontiguousarray(zd)
        assert zd.shape == (B, K, V) and zd.dtype == zt.dtype
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, K)
    ln = np.ascontiguousarray(lengths, dtype=np.int32).reshape(B)
    tp = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    rid = None if row_ids is None else np.ascontiguousarray(row_ids, dtype=np.int64).reshape(B)
    alt = np.zeros((B, K + 1, 4), dtype=np.int32)
    st = lib().oracle_verify_window(_p(zt), _p(zd), dt, B, K, V, _p(tok), _p(ln), _p(tp),
                                    ctypes.c_uint64(seed & (2**64 - 1)), int(row_base), _p(rid),
                                    float(w_acc), float(w_cdf), _p(alt), int(nthreads))
    if st < 0:
        raise ValueError("oracle_verify_window: bad arguments")
    return alt, st


def verify_window_row_u(zt, zd, x, L, T, u_acc, u_res, w_acc, w_cdf):
    """One row of :func:`verify_window` with fp64 logits and injected
    uniforms (zt [K+1, V], zd [K, V] or None).  Returns alt [K+1, 4]."""
    zt = np.ascontiguousarray(zt, dtype=np.float64)
    K1, V = zt.shape
    K = K1 - 1
    zd_a = None if zd is None else np.ascontiguousarray(zd, dtype=np.float64)
    x = np.ascontiguousarray(x, dtype=np.int32).reshape(K)
    ua = np.ascontiguousarray(u_acc, dtype=np.float64).reshape(-1)
    ur = np.ascontiguousarray(u_res, dtype=np.float64).reshape(-1)
    assert ua.size >= K + 1 and ur.size >= K + 1
    alt = np.zeros((K + 1, 4), dtype=np.int32)
    r = lib().oracle_verify_window_row_u(_p(zt), _p(zd_a), K, V, _p(x), int(L), float(T),
                                         _p(ua), _p(ur), float(w_acc), float(w_cdf), _p(alt))
    if r < 0:
        raise ValueError("oracle_verify_window_row_u: bad arguments")
    return alt


def stats(z, temperature, nthreads=0):
    """Per-vector (m, Sigma, argmax) of z [..., V] (float32 or bf16 bits) at a
    per-vector temperature broadcastable to z.shape[:-1]."""
    z = np.ascontiguousarray(z)
    V = z.shape[-1]
    n = int(np.prod(z.shape[:-1]))
    T = np.ascontiguousarray(np.broadcast_to(np.asarray(temperature, dtype=np.float32),
                                             z.shape[:-1])).reshape(n)
    m = np.zeros(n, dtype=np.float64)
    s = np.zeros(n, dtype=np.float64)
    am = np.zeros(n, dtype=np.int32)
    lib().oracle_stats_batch(_p(z), _dtype_code(z), n, V, _p(T), _p(m), _p(s), _p(am),
                             int(nthreads))
    shp = z.shape[:-1]
    return m.reshape(shp), s.reshape(shp), am.reshape(shp)


def schedule(conf, tau):
    """Verify lengths from confidences conf [B, K] (float32) and threshold tau.
    Returns (lengths [B] int32, S [B, K] fp64, smallest |S_i - tau|)."""
    c = np.ascontiguousarray(conf, dtype=np.float32)
    B, K = c.shape
    ln = np.zeros(B, dtype=np.int32)
    S = np.zeros((B, K), dtype=np.float64)
    closest = lib().oracle_schedule(_p(c), B, K, float(tau), _p(ln), _p(S))
    return ln, S, closest


def schedule_admit(conf, speed):
    """Hardware-aware admission: candidates sorted by prefix survival are
    admitted while (expected emitted tokens) x speed[batch tokens] rises.
    conf [B, K] float32, speed [n] float32 (steps/s at n verified tokens).
    Returns (lengths [B] int32, tau, k admitted, f [k_evaluated+1] fp64)."""
    c = np.ascontiguousarray(conf, dtype=np.float32)
    B, K = c.shape
    sp = np.ascontiguousarray(speed, dtype=np.float32).reshape(-1)
    ln = np.zeros(B, dtype=np.int32)
    tau = np.zeros(1, dtype=np.float64)
    f = np.full(B * K + 1, np.nan, dtype=np.float64)
    k = lib().oracle_schedule_admit(_p(c), B, K, _p(sp), sp.size, _p(ln), _p(tau), _p(f))
    return ln, float(tau[0]), int(k), f


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def sts_fit(logits, accept, tmin=1e-2, tmax=1e2):
    """Per-position temperature scaling of the confidence head on held-out
    blocks: logits [N, K] float32 (confidence = sigmoid), accepted lengths
    [N] int32 (position i observed iff i <= a, survived iff i < a; a < 0
    skips the block).  Returns (T [K] fp64, (ece_before, ece_after),
    observed count)."""
    l = np.ascontiguousarray(logits, dtype=np.float32)
    N, K = l.shape
    a = np.ascontiguousarray(accept, dtype=np.int32).reshape(-1)
    T = np.zeros(K, dtype=np.float64)
    ece = np.zeros(2, dtype=np.float64)
    n = lib().oracle_sts_fit(_p(l), _p(a), N, K, ctypes.c_double(tmin), ctypes.c_double(tmax),
                             _p(T), _p(ece))
    if n < 0:
        raise ValueError("bad arguments")
    return T, (float(ece[0]), float(ece[1])), int(n)
