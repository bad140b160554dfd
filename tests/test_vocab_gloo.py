"""Vocabulary-parallel verification on CPU ranks (gloo): the exchanges of
``vocab_parallel`` -- all-gather in rank order and the max-reduce of the
tokens -- around a plain fp64 numpy model of the three per-slice steps,
reproduce the oracle's result on the unsplit vocabulary.

The numpy model restates, slice by slice, what the kernels compute: the
slice's (max, sum of exp) and draft-token logit; the merged normalisers and
accept tests, identical on every rank; the slice's draw mass; and the draw
by the rank whose slice holds the CDF target.  It checks the decomposition
and the exchange protocol on 2 and 3 ranks; the kernels themselves are
checked against the oracle on the GPU (test_gpu_vocab.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verification_93_b200.vocab_parallel import (
    gather_in_rank_order, reduce_tokens, shard_vocab)


def test_shard_vocab_partition():
    for V in (3, 1000, 129280):
        for world in (1, 2, 3, 8):
            if V < world:
                continue
            spans = [shard_vocab(V, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == V
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(b - a for a, b in spans) <= -(-V // world)
    with pytest.raises(ValueError):
        shard_vocab(2, 3, 0)


def _slice_stats(zt, zd, v0, tokens, lengths, T):
    """Per (row, slot): (m, Sigma, z_x, own) of the slice; greedy rows
    (max, 0, 0, global argmax).  Slots: target 0..K, draft K+1..2K."""
    B, K1, _ = zt.shape
    K = K1 - 1
    out = np.zeros((B, 2 * K + 1, 4))
    out[:, :, 0] = -np.inf
    for b in range(B):
        for slot in range(2 * K + 1):
            i = slot if slot <= K else slot - K - 1
            z = zt[b, i] if slot <= K else (None if zd is None else zd[b, i])
            if z is None or (slot > K and (T[b] == 0 or i >= lengths[b])) or i > lengths[b]:
                continue
            m = z.max()
            if T[b] == 0:
                out[b, slot] = (m, 0.0, 0.0, v0 + int(np.argmax(z)))
                continue
            s = np.exp((z - m) / T[b]).sum() if m > -np.inf else 0.0
            zx, own = 0.0, 0.0
            if i < lengths[b]:
                xl = tokens[b, i] - v0
                if 0 <= xl < len(z):
                    zx, own = z[xl], 1.0
            out[b, slot] = (m, s, zx, own)
    return out


def _merge(parts, T):
    """Rank-order merge of one slot's partials -> (m, Sigma, z_x, argmax)."""
    m = max(p[0] for p in parts)
    if T == 0:
        best = min(int(p[3]) for p in parts if p[0] == m)
        return m, 1.0, None, best
    s = sum(p[1] * np.exp((p[0] - m) / T) for p in parts if p[0] > -np.inf)
    zx = next((p[2] for p in parts if p[3] == 1.0), -np.inf)
    return m, s, zx, None


def _decide(stats_all, world, zt, zd, v0, tokens, lengths, T, seed, oracle):
    """Accept tests on the merged normalisers and this slice's draw mass."""
    B, K1, _ = zt.shape
    K = K1 - 1
    per = stats_all.reshape(world, B, 2 * K + 1, 4)
    out = np.full((B, K1), -1, np.int32)
    acc = np.zeros(B, np.int32)
    draws = {}
    mass = np.zeros((B, 2))
    for b in range(B):
        L, t = int(lengths[b]), float(T[b])
        merged = {s: _merge([per[r, b, s] for r in range(world)], t)
                  for s in list(range(L + 1)) + ([K + 1 + i for i in range(L)]
                                                 if zd is not None and t > 0 else [])}
        j = L
        for i in range(L):
            x = tokens[b, i]
            if t == 0:
                ok = x == merged[i][3]
            else:
                mt, st, zx, _ = merged[i]
                p = np.exp((zx - mt) / t) / st
                q = 1.0
                if zd is not None:
                    md, sd, zdx, _ = merged[K + 1 + i]
                    q = np.exp((zdx - md) / t) / sd
                if p == 0:
                    ok = False
                elif q == 0:
                    ok = True
                else:
                    ok = oracle.uniform(seed, b, i, 0) < min(1.0, p / q)
            if not ok:
                j = i
                break
        acc[b] = j
        out[b, :j] = tokens[b, :j]
        if t == 0:
            out[b, j] = merged[j][3]
            continue
        mt, st, _, _ = merged[j]
        p = np.exp((zt[b, j] - mt) / t)
        if j < L and zd is not None:
            md, sd, _, _ = merged[K + 1 + j]
            w = np.maximum(p / st - np.exp((zd[b, j] - md) / t) / sd, 0.0)
        elif j < L:
            w = p.copy()
            xl = tokens[b, j] - v0
            if 0 <= xl < len(w):
                w[xl] = 0.0
        else:
            w = p
        draws[b] = (j, w, p)
        mass[b] = (w.sum(), p.sum())
    return out, acc, draws, mass


def _draw(out, mass_all, world, rank, draws, v0, seed, oracle):
    B = out.shape[0]
    per = mass_all.reshape(world, B, 2)
    for b, (j, w, p) in draws.items():
        col = 0 if per[:, b, 0].sum() > 0 else 1
        tgt = oracle.uniform(seed, b, j, 1) * per[:, b, col].sum()
        cum = 0.0
        for r in range(world):
            if cum + per[r, b, col] > tgt:
                if r == rank:
                    c = np.cumsum(w if col == 0 else p)
                    out[b, j] = v0 + int(np.argmax(c > tgt - cum))
                break
            cum += per[r, b, col]


def _worker(rank, world, port, path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from speculative_decoding_verification_93_b200 import workloads
        from speculative_decoding_verification_93_b200.workloads import to_host_logits
        bt = workloads.random_small(20, 4, 301, dtype=torch.float32, seed=9,
                                    temps=(0.0, 0.6, 1.0))
        zt, zd = to_host_logits(bt.zt), to_host_logits(bt.zd)
        tokens, lengths, T = bt.tokens.numpy(), bt.lengths.numpy(), bt.temperature.numpy()
        v0, v1 = shard_vocab(301, world, rank)
        ok = True
        for zdx in (zd, None):
            seed = 31
            zt_s = zt[:, :, v0:v1].astype(np.float64)
            zd_s = None if zdx is None else zdx[:, :, v0:v1].astype(np.float64)
            st = torch.from_numpy(_slice_stats(zt_s, zd_s, v0, tokens, lengths, T))
            st_all = torch.empty((world * st.shape[0],) + tuple(st.shape[1:]), dtype=st.dtype)
            gather_in_rank_order(st, st_all)
            out, acc, draws, mass = _decide(st_all.numpy(), world, zt_s, zd_s, v0, tokens,
                                            lengths, T, seed, oracle)
            m_all = torch.empty(world * mass.shape[0], 2, dtype=torch.float64)
            gather_in_rank_order(torch.from_numpy(mass), m_all)
            _draw(out, m_all.numpy(), world, rank, draws, v0, seed, oracle)
            tok = torch.from_numpy(out)
            reduce_tokens(tok)
            o_tok, o_acc, diag, _ = oracle.verify(zt, zdx, tokens, lengths, T, seed, nthreads=1)
            tie = (diag[:, 0] < 1e-9) | (diag[:, 1] < 1e-9)
            same = (acc == o_acc) & np.all(tok.numpy() == o_tok, axis=1)
            ok &= bool(np.all(same | tie)) and int(tie.sum()) <= 1
        flags = torch.tensor([1 if ok else 0], dtype=torch.int32)
        dist.all_reduce(flags, op=dist.ReduceOp.MIN)
        if rank == 0:
            with open(path, "w") as f:
                f.write("ok" if flags.item() == 1 else "mismatch")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_reproduce_unsplit_vocabulary(tmp_path, world):
    path = str(tmp_path / "result.txt")
    mp.start_processes(_worker, args=(world, _free_port(), path), nprocs=world, join=True,
                       start_method="spawn")
    assert open(path).read() == "ok"


def test_exchanges_without_a_process_group():
    """One rank: the gather copies (or aliases) and the reduction is a no-op."""
    local = torch.arange(6, dtype=torch.float32).reshape(3, 2)
    out = torch.zeros(3, 2)
    assert torch.equal(gather_in_rank_order(local, out), local)
    assert gather_in_rank_order(local, local) is local
    tok = torch.tensor([[3, -1], [-1, 5]], dtype=torch.int32)
    assert torch.equal(reduce_tokens(tok.clone()), tok)


def test_verifier_buffers_and_slice_checks_on_cpu():
    """Buffer sizing of one rank (no process group) and the slice
    description's argument checks; no kernel runs."""
    import speculative_decoding_verification_93_b200 as sv
    from speculative_decoding_verification_93_b200.vocab_parallel import VocabParallelVerifier
    v = VocabParallelVerifier(256, 8, 129280, torch.bfloat16, "cpu")
    assert (v.world, v.rank, v.v0, v.Vs) == (1, 0, 0, 129280)
    assert v.stats_local.numel() == 256 * 17 * 4 * 16          # four 64 KB chunks per vector
    assert v.stats_all is v.stats_local and v.mass_all is v.mass_local
    assert v.workspace.numel() > 256 * 2 * 506 * 4             # two segment tables per row
    with pytest.raises(TypeError):
        VocabParallelVerifier(4, 2, 100, torch.float16, "cpu")
    zt = torch.zeros(2, 3, 50)
    d = sv.vp_slice(zt, torch.zeros(2, 2, 50), 100, 50, 2, 1)
    assert (d.B, d.K, d.V, d.v0, d.Vs, d.nshards, d.shard) == (2, 2, 100, 50, 50, 2, 1)
    with pytest.raises(TypeError):
        sv.vp_slice(zt, torch.zeros(2, 2, 49), 100, 50, 2, 1)     # draft slice of another width
    with pytest.raises(TypeError):
        sv.vp_slice(zt.double(), None, 100, 50, 2, 1)             # unsupported dtype
    with pytest.raises(ValueError):
        v.slice_of(torch.zeros(256, 9, 100, dtype=torch.bfloat16), None)
