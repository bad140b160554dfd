"""GPU vs oracle parity of vocabulary-parallel verification (sv_vp_stats,
sv_vp_decide, sv_vp_draw) through the C ABI.

N ranks are emulated on one GPU: each rank's slice is its own contiguous
tensor and its three steps are separate launches that never wait on one
another; the exchanges between them (all-gather in rank order, max-reduce of
the tokens) are done here with torch, exactly as the collectives would
deliver them.  Every rank must report the same accept lengths, exactly one
rank must write each drawn token, and the merged result must match the
oracle on the unsplit vocabulary outside the tie windows."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200 import workloads
from speculative_decoding_verification_93_b200.vocab_parallel import shard_vocab
from speculative_decoding_verification_93_b200.workloads import to_host_logits
from _parity import check_batch, check_structure, compare, gpu_schedule, oracle_verify

pytestmark = pytest.mark.gpu


def vp_emulated(zt, zd, tokens, lengths, temperature, seed, nshards, row_base=0, norms=False):
    B, K1, V = zt.shape
    K = K1 - 1
    dev = zt.device
    ranks = []
    for r in range(nshards):
        v0, v1 = shard_vocab(V, nshards, r)
        zt_r = zt[:, :, v0:v1].contiguous()
        zd_r = None if zd is None else zd[:, :, v0:v1].contiguous()
        ranks.append((zt_r, zd_r, sv.vp_slice(zt_r, zd_r, V, v0, nshards, r)))
    nst = sv.sv_vp_stats_bytes(ranks[0][2])
    assert nst > 0 and all(sv.sv_vp_stats_bytes(d) == nst for _, _, d in ranks)
    stats_all = torch.empty(nshards * nst, dtype=torch.uint8, device=dev)
    for r, (_, _, d) in enumerate(ranks):
        sv.sv_vp_stats(d, tokens, lengths, temperature, stats_all[r * nst:(r + 1) * nst])
    mass_all = torch.empty(nshards * B, 2, dtype=torch.float32, device=dev)
    outs = []
    for r, (_, _, d) in enumerate(ranks):
        ws = torch.randint(0, 255, (sv.sv_vp_workspace_bytes(d),), dtype=torch.uint8,
                           device=dev)
        ot = torch.full((B, K1), -7, dtype=torch.int32, device=dev)
        oa = torch.full((B,), -7, dtype=torch.int32, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        nm = torch.full((B, 2 * K + 1, 2), float("nan"), device=dev) if norms else None
        sv.sv_vp_decide(d, stats_all, tokens, lengths, temperature, seed, ot, oa,
                        mass_all[r * B:(r + 1) * B], ws, status=st, norm_out=nm,
                        row_base=row_base)
        outs.append((ot, oa, st, ws, nm))
    drawn = []
    for r, (_, _, d) in enumerate(ranks):
        ot, oa, st, ws, _ = outs[r]
        before = ot.clone()
        sv.sv_vp_draw(d, mass_all, ot, ws, status=st)
        drawn.append(ot != before)
    torch.cuda.synchronize()
    acc = [o[1].cpu().numpy() for o in outs]
    for a in acc[1:]:
        assert np.array_equal(a, acc[0]), "ranks disagree on accept lengths"
    wrote = torch.stack(drawn).sum(0).cpu().numpy()
    assert wrote.max(initial=0) <= 1, "two ranks drew the same token"
    tokens_all = torch.stack([o[0] for o in outs]).amax(0).cpu().numpy()
    status = 0
    for o in outs:
        status |= int(o[2].item())
    return dict(tokens=tokens_all, accept=acc[0], status=status, wrote=wrote,
                norms=None if not norms else outs[0][4].cpu().numpy(),
                all_norms=None if not norms else [o[4].cpu().numpy() for o in outs])


def _cuda(batch):
    for name in ("zt", "zd", "tokens", "temperature", "conf", "lengths"):
        t = getattr(batch, name)
        if t is not None:
            setattr(batch, name, t.cuda())
    return batch


@pytest.mark.parametrize("nshards", [1, 2, 3, 4])
def test_c0_matches_oracle(nshards):
    b = _cuda(workloads.make_batch("c0", device="cpu"))
    for seed in (0, 1, 2):
        g = vp_emulated(b.zt, b.zd, b.tokens, b.lengths, b.temperature, seed, nshards)
        o = oracle_verify(b.zt, b.zd, b.tokens, b.lengths.cpu().numpy(), b.temperature, seed)
        check_structure(g, b.tokens.cpu().numpy(), b.lengths.cpu().numpy())
        res = compare(g, o)
        assert g["status"] == 0 and res["ties"] == 0


CASES = [
    # V, dtype, K, B, nshards: ragged slices (Vs not a multiple of 16 bytes,
    # slices out of 16-byte phase with each other), one token per slice,
    # several chunks and segments per slice.
    (5, torch.float32, 4, 32, 5), (7, torch.bfloat16, 8, 32, 3), (33, torch.float32, 5, 32, 4),
    (1000, torch.bfloat16, 4, 32, 8), (1001, torch.bfloat16, 6, 32, 3),
    (1003, torch.float32, 2, 24, 2), (8193, torch.bfloat16, 7, 16, 5),
    (20011, torch.float32, 3, 12, 8), (65543, torch.bfloat16, 2, 8, 1),
    (65543, torch.bfloat16, 2, 8, 6), (200003, torch.float32, 2, 6, 2),
]


@pytest.mark.parametrize("V,dtype,K,B,nshards", CASES)
def test_ragged_slices_match_oracle(V, dtype, K, B, nshards):
    b = _cuda(workloads.random_small(B, K, V, dtype=dtype, seed=V + K + nshards,
                                     temps=(0.0, 0.6, 1.0, 2.5)))
    total = dict(rows=0, tie_mismatches=0)
    for seed in (7, 8):
        for zd in (b.zd, None):
            g = vp_emulated(b.zt, zd, b.tokens, b.lengths, b.temperature, seed, nshards)
            ln = b.lengths.cpu().numpy()
            o = oracle_verify(b.zt, zd, b.tokens, ln, b.temperature, seed)
            check_structure(g, b.tokens.cpu().numpy(), ln)
            r = compare(g, o)
            total["rows"] += r["rows"]
            total["tie_mismatches"] += r["tie_mismatches"]
            assert g["status"] & ~(sv.SV_NOTE_CDF_FALLBACK | sv.SV_NOTE_ZERO_RESIDUAL) == 0
            # sampled rows: exactly one rank drew; greedy rows: none did
            T = b.temperature.cpu().numpy()
            assert np.array_equal(g["wrote"].sum(1), (T > 0).astype(np.int64))
    assert total["tie_mismatches"] <= max(2, total["rows"] // 50)


@pytest.mark.parametrize("B,V,dtype,nshards", [(1025, 1000, torch.bfloat16, 2),
                                              (2100, 517, torch.float32, 3)])
def test_many_rows(B, V, dtype, nshards):
    """Thousands of rows (grids of tens of thousands of stats CTAs, most of
    them for slots no row reads) against the oracle."""
    b = _cuda(workloads.random_small(B, 3, V, dtype=dtype, seed=B + V, temps=(0.0, 0.6, 1.0, 2.5)))
    g = vp_emulated(b.zt, b.zd, b.tokens, b.lengths, b.temperature, 11, nshards)
    ln = b.lengths.cpu().numpy()
    o = oracle_verify(b.zt, b.zd, b.tokens, ln, b.temperature, 11)
    check_structure(g, b.tokens.cpu().numpy(), ln)
    r = compare(g, o)
    assert g["status"] & ~(sv.SV_NOTE_CDF_FALLBACK | sv.SV_NOTE_ZERO_RESIDUAL) == 0
    assert r["tie_mismatches"] <= max(2, r["rows"] // 50)


@pytest.mark.parametrize("V,dtype,nshards", [(1000, torch.float32, 3),
                                             (129280, torch.bfloat16, 8),
                                             (20011, torch.float32, 5)])
def test_merged_normalisers_match_oracle(V, dtype, nshards):
    """Every rank holds the same merged (m, Sigma): m bit-exact, Sigma within
    1e-5 relative of the oracle, for target slots 0..L and draft slots
    0..L-1 of sampled rows; slots that are not read stay untouched."""
    B, K = 16, 4
    b = _cuda(workloads.random_small(B, K, V, dtype=dtype, seed=3, temps=(0.0, 0.6, 1.0, 1.7)))
    g = vp_emulated(b.zt, b.zd, b.tokens, b.lengths, b.temperature, 5, nshards, norms=True)
    for other in g["all_norms"][1:]:
        assert np.array_equal(np.nan_to_num(other, nan=-7.0), np.nan_to_num(g["norms"], nan=-7.0))
    st = g["norms"]
    T = b.temperature.cpu().numpy()
    ln = b.lengths.cpu().numpy()
    mt, St, _ = oracle.stats(to_host_logits(b.zt), T[:, None])
    md, Sd, _ = oracle.stats(to_host_logits(b.zd), T[:, None])
    for r in range(B):
        L = ln[r]
        for i in range(K + 1):
            if i <= L:
                assert st[r, i, 0] == mt[r, i]
                if T[r] > 0:
                    assert abs(st[r, i, 1] - St[r, i]) <= 1e-5 * St[r, i]
            else:
                assert np.isnan(st[r, i, 0])
        for i in range(K):
            if T[r] > 0 and i < L:
                assert st[r, K + 1 + i, 0] == md[r, i]
                assert abs(st[r, K + 1 + i, 1] - Sd[r, i]) <= 1e-5 * Sd[r, i]
            else:
                assert np.isnan(st[r, K + 1 + i, 0])


def test_edge_cases_and_invalid_rows():
    dev = "cuda"
    B, K, V = 12, 3, 300
    zt = torch.zeros(B, K + 1, V, device=dev)
    zd = torch.zeros(B, K, V, device=dev)
    zt[:, :, 50:] = float("-inf")
    zd[:, :, 100:] = float("-inf")
    zt[6:, :, :] = torch.randn(B - 6, K + 1, V, device=dev)
    tokens = torch.randint(0, 50, (B, K), dtype=torch.int32, device=dev)
    temp = torch.tensor([1.0, 1e-6, 0.0, 2.0] * 3, device=dev)
    for L in (0, 1, K):
        ln = torch.full((B,), L, dtype=torch.int32, device=dev)
        for nshards in (1, 4, 7):
            g = vp_emulated(zt, zd, tokens, ln, temp, 3, nshards)
            o = oracle_verify(zt, zd, tokens, ln.cpu().numpy(), temp, 3)
            check_structure(g, tokens.cpu().numpy(), ln.cpu().numpy())
            compare(g, o)
            fin = g["tokens"][np.arange(B), g["accept"]]
            assert np.all(fin[:6] < 50)
    # invalid rows are marked on every rank, the rest are unaffected
    B, K, V = 6, 3, 64
    zt = torch.randn(B, K + 1, V, device=dev)
    zd = torch.randn(B, K, V, device=dev)
    tokens = torch.randint(0, V, (B, K), dtype=torch.int32, device=dev)
    tokens[1, 0] = V
    tokens[5, 2] = -3
    ln = torch.tensor([3, 3, 4, 1, -1, 2], dtype=torch.int32, device=dev)
    temp = torch.tensor([1.0, 1.0, 1.0, float("nan"), 1.0, 1.0], device=dev)
    g = vp_emulated(zt, zd, tokens, ln, temp, 1, 3)
    assert g["status"] == (sv.SV_ROW_BAD_TOKEN | sv.SV_ROW_BAD_LENGTH
                           | sv.SV_ROW_BAD_TEMPERATURE)
    assert list(g["accept"][[1, 2, 3, 4]]) == [-1, -1, -1, -1]
    assert np.all(g["tokens"][[1, 2, 3, 4]] == -1)
    o = oracle_verify(zt, zd, tokens, ln.cpu().numpy(), temp, 1)
    compare(g, o)


def test_row_base_and_determinism():
    b = _cuda(workloads.random_small(32, 4, 5000, dtype=torch.bfloat16, seed=4, temps=(0.0, 1.0)))
    g1 = vp_emulated(b.zt, b.zd, b.tokens, b.lengths, b.temperature, 99, 4, row_base=1000)
    g2 = vp_emulated(b.zt, b.zd, b.tokens, b.lengths, b.temperature, 99, 4, row_base=1000)
    assert np.array_equal(g1["tokens"], g2["tokens"])
    o = oracle_verify(b.zt, b.zd, b.tokens, b.lengths.cpu().numpy(), b.temperature, 99,
                      row_base=1000)
    compare(g1, o)


@pytest.mark.parametrize("nshards", [1, 8])
def test_c2_full_split(nshards):
    """B = 256, K = 8, V = 129280 bf16 with lengths from the schedule, the
    vocabulary split over 1 or 8 ranks."""
    b = workloads.make_batch("c2", device="cuda")
    ln = gpu_schedule(b.conf, b.tau)
    g = vp_emulated(b.zt, b.zd, b.tokens, ln, b.temperature, 0, nshards)
    check_structure(g, b.tokens.cpu().numpy(), ln.cpu().numpy())
    res = check_batch(b, ln, g, 0)
    assert g["status"] & ~(sv.SV_NOTE_CDF_FALLBACK | sv.SV_NOTE_ZERO_RESIDUAL) == 0
    assert res["invalid"] == 0 and res["rows"] == 256
    assert res["window_valid"] <= max(2, res["rows"] // 50), res


@pytest.mark.parametrize("V,dtype,K,B,nshards", [
    (1000, torch.float32, 4, 16, 40),      # more ranks than a warp holds: masses read 32 at a time
    (2003, torch.bfloat16, 3, 16, 77),
    (3000, torch.bfloat16, 40, 12, 3),     # accept tests in two rounds of 32 positions
    (513, torch.float32, 64, 8, 5),        # the largest K
])
def test_many_ranks_and_long_blocks(V, dtype, K, B, nshards):
    b = _cuda(workloads.random_small(B, K, V, dtype=dtype, seed=V + K, noise=0.05,
                                     temps=(0.0, 0.8, 1.0)))
    total = dict(rows=0, tie_mismatches=0)
    longest = 0
    for seed in (1, 2):
        for zd in (b.zd, None):
            g = vp_emulated(b.zt, zd, b.tokens, b.lengths, b.temperature, seed, nshards)
            ln = b.lengths.cpu().numpy()
            o = oracle_verify(b.zt, zd, b.tokens, ln, b.temperature, seed)
            check_structure(g, b.tokens.cpu().numpy(), ln)
            r = compare(g, o)
            total["rows"] += r["rows"]
            total["tie_mismatches"] += r["tie_mismatches"]
            if zd is not None:
                longest = max(longest, int(g["accept"].max()))
    assert total["tie_mismatches"] <= max(2, total["rows"] // 50)
    # drafts close to the target (noise 0.05) keep long blocks alive, so the
    # second round of accept tests (positions 32..) is exercised
    if K > 32 and b.lengths.max().item() > 33:
        assert longest > 32


def test_verifier_class_single_rank():
    """VocabParallelVerifier without a process group (one rank, collectives
    skipped): the public orchestration path, reused across steps."""
    from speculative_decoding_verification_93_b200.vocab_parallel import VocabParallelVerifier
    b = _cuda(workloads.random_small(24, 5, 4099, dtype=torch.bfloat16, seed=21,
                                     temps=(0.0, 0.7, 1.0)))
    vpv = VocabParallelVerifier(24, 5, 4099, torch.bfloat16, "cuda")
    assert (vpv.world, vpv.rank, vpv.v0, vpv.Vs) == (1, 0, 0, 4099)
    ln = b.lengths.cpu().numpy()
    for seed in (3, 4):
        ot = torch.full((24, 6), -7, dtype=torch.int32, device="cuda")
        oa = torch.full((24,), -7, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        vpv.step(b.zt, b.zd, b.tokens, b.lengths, b.temperature, seed, ot, oa, status=st)
        torch.cuda.synchronize()
        g = dict(tokens=ot.cpu().numpy(), accept=oa.cpu().numpy(), status=int(st.item()))
        o = oracle_verify(b.zt, b.zd, b.tokens, ln, b.temperature, seed)
        check_structure(g, b.tokens.cpu().numpy(), ln)
        compare(g, o)
    with pytest.raises(ValueError):
        vpv.slice_of(b.zt[:, :, :100].contiguous(), None)
