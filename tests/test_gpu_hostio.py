"""sv_verify_host: inputs and outputs in host memory, only the scheduled
logit runs copied to the device.  Its results must equal sv_schedule +
sv_verify on device copies of the same inputs bit for bit, with the device
workspace filled with random bytes beforehand (so a read of any unscheduled
position would show), and the host-to-device byte count must be exactly the
scheduled runs plus the small arrays."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200 import workloads
from _parity import gpu_schedule, gpu_verify

pytestmark = pytest.mark.gpu


def _host_run(b, tau, seed, with_draft=True, row_base=0, levelwise=False):
    B, K1, V = b.zt.shape
    K = K1 - 1
    dt = sv.SV_BF16 if b.zt.dtype == torch.bfloat16 else sv.SV_F32
    host = lambda t: t.detach().cpu().contiguous().pin_memory()
    zt, conf, tok, temp = host(b.zt), host(b.conf), host(b.tokens), host(b.temperature)
    zd = host(b.zd) if with_draft else None
    ot = torch.full((B, K1), -7, dtype=torch.int32).pin_memory()
    oa = torch.full((B,), -7, dtype=torch.int32).pin_memory()
    ln = torch.full((B,), -7, dtype=torch.int32).pin_memory()
    st = torch.full((1,), -7, dtype=torch.int32).pin_memory()
    n = sv.sv_verify_host_workspace_bytes(B, K, V, dt)
    ws = torch.randint(0, 255, (n,), dtype=torch.uint8, device="cuda")
    h2d = sv.sv_verify_host(zt, zd, conf, tau, tok, temp, seed, ot, oa, ln, ws, status=st,
                            row_base=row_base, levelwise=levelwise)
    torch.cuda.synchronize()
    return ot.numpy(), oa.numpy(), ln.numpy(), int(st.item()), h2d


def _device_run(b, tau, seed, with_draft=True, row_base=0):
    ln = gpu_schedule(b.conf.cuda(), tau)
    g = gpu_verify(b.zt.cuda(), b.zd.cuda() if with_draft else None, b.tokens.cuda(), ln,
                   b.temperature.cuda(), seed, row_base=row_base)
    return g["tokens"], g["accept"], ln.cpu().numpy(), g["status"]


def _expected_h2d(b, lengths, with_draft):
    B, K1, V = b.zt.shape
    K = K1 - 1
    es = b.zt.element_size()
    T = b.temperature.cpu().numpy()
    n = int(sum((L + 1) * V * es for L in lengths))
    if with_draft:
        n += int(sum(L * V * es for L, t in zip(lengths, T) if t > 0))
    return n + B * K * 8 + B * 4


def _expected_h2d_levelwise(b, lengths, accept, with_draft, scheduled=True):
    """Target 0..a and draft 0..min(a, L-1) of sampled rows (what the outcome
    depends on), plus for a row that rejects at a < L the next position,
    copied before the rejection is known (target a+1; draft a+1 if a+1 < L);
    the small arrays.  The lengths of each level are computed on the device."""
    B, K1, V = b.zt.shape
    K = K1 - 1
    es = b.zt.element_size()
    T = b.temperature.cpu().numpy()
    n = int(sum((a + 2 if a < L else L + 1) * V * es for a, L in zip(accept, lengths)))
    if with_draft:
        n += int(sum(min(a + 2, L) * V * es for a, L, t in zip(accept, lengths, T) if t > 0))
    return n + B * K * 4 + B * 4 + (B * K * 4 if scheduled else 0)


@pytest.mark.parametrize("levelwise", [False, True])
@pytest.mark.parametrize("V,dtype,K,B,with_draft", [
    (1000, torch.float32, 4, 32, True), (1001, torch.bfloat16, 6, 48, True),
    (4099, torch.bfloat16, 3, 40, False), (33, torch.float32, 8, 64, True)])
def test_host_path_equals_device_path(V, dtype, K, B, with_draft, levelwise):
    b = workloads.random_small(B, K, V, dtype=dtype, seed=V + K, temps=(0.0, 0.6, 1.0))
    for tau, seed in ((0.3, 5), (0.05, 6), (0.9, 7)):
        ht, ha, hl, hs, h2d = _host_run(b, tau, seed, with_draft, row_base=11,
                                        levelwise=levelwise)
        dt_, da, dl, ds = _device_run(b, tau, seed, with_draft, row_base=11)
        assert np.array_equal(hl, dl)
        assert np.array_equal(ha, da) and np.array_equal(ht, dt_)
        if levelwise:
            assert hs & ~sv.SV_NOTE_CDF_FALLBACK == ds & ~sv.SV_NOTE_CDF_FALLBACK
            assert h2d == _expected_h2d_levelwise(b, hl, ha, with_draft)
        else:
            assert hs == ds
            assert h2d == _expected_h2d(b, hl, with_draft)


@pytest.mark.parametrize("levelwise", [False, True])
def test_host_path_full_size_c2(levelwise):
    b = workloads.make_batch("c2", device="cuda")
    ht, ha, hl, hs, h2d = _host_run(b, b.tau, 0, levelwise=levelwise)
    dt_, da, dl, ds = _device_run(b, b.tau, 0)
    assert np.array_equal(hl, dl) and np.array_equal(ha, da) and np.array_equal(ht, dt_)
    assert ds == 0 and hs & ~sv.SV_NOTE_CDF_FALLBACK == 0
    full = (b.zt.numel() + b.zd.numel()) * 2
    if levelwise:
        assert h2d == _expected_h2d_levelwise(b, hl, ha, True) and h2d < 0.35 * full
    else:
        assert hs == 0
        assert h2d == _expected_h2d(b, hl, True) and h2d < 0.6 * full


def test_levelwise_invalid_rows():
    """Invalid lengths, temperatures and tokens end as -1 rows with their bits,
    exactly as on the device path."""
    b = workloads.random_small(12, 4, 500, dtype=torch.float32, seed=8, temps=(0.0, 1.0))
    b.lengths = torch.tensor([4, -1, 2, 5, 3, 0, 4, 1, 2, 3, 4, 4], dtype=torch.int32)
    b.temperature[6] = float("nan")
    b.tokens[9, 1] = 500
    B, K1, V = b.zt.shape
    host = lambda t: t.detach().cpu().contiguous().pin_memory()
    ln = host(b.lengths)
    ot = torch.empty((B, K1), dtype=torch.int32).pin_memory()
    oa = torch.empty((B,), dtype=torch.int32).pin_memory()
    st = torch.zeros(1, dtype=torch.int32).pin_memory()
    ws = torch.randint(0, 255, (sv.sv_verify_host_workspace_bytes(B, K1 - 1, V, sv.SV_F32),),
                       dtype=torch.uint8, device="cuda")
    sv.sv_verify_host(host(b.zt), host(b.zd), None, 0.0, host(b.tokens), host(b.temperature), 4,
                      ot, oa, ln, ws, status=st, levelwise=True)
    torch.cuda.synchronize()
    g = gpu_verify(b.zt.cuda(), b.zd.cuda(), b.tokens.cuda(), b.lengths.cuda(),
                   b.temperature.cuda(), 4)
    assert np.array_equal(oa.numpy(), g["accept"]) and np.array_equal(ot.numpy(), g["tokens"])
    assert list(oa.numpy()[[1, 3, 6, 9]]) == [-1, -1, -1, -1]
    assert int(st.item()) & 7 == g["status"] & 7 == 7


def test_host_path_with_given_lengths():
    """conf None: the caller's lengths are used, no schedule runs."""
    b = workloads.random_small(24, 5, 2003, dtype=torch.bfloat16, seed=3, temps=(0.0, 1.0))
    B, K1, V = b.zt.shape
    host = lambda t: t.detach().cpu().contiguous().pin_memory()
    ln = host(b.lengths)
    ot = torch.empty((B, K1), dtype=torch.int32).pin_memory()
    oa = torch.empty((B,), dtype=torch.int32).pin_memory()
    ws = torch.randint(0, 255, (sv.sv_verify_host_workspace_bytes(B, K1 - 1, V, sv.SV_BF16),),
                       dtype=torch.uint8, device="cuda")
    h2d = sv.sv_verify_host(host(b.zt), host(b.zd), None, 0.0, host(b.tokens),
                            host(b.temperature), 9, ot, oa, ln, ws)
    torch.cuda.synchronize()
    g = gpu_verify(b.zt.cuda(), b.zd.cuda(), b.tokens.cuda(), b.lengths.cuda(),
                   b.temperature.cuda(), 9)
    assert np.array_equal(oa.numpy(), g["accept"]) and np.array_equal(ot.numpy(), g["tokens"])
    assert np.array_equal(ln.numpy(), b.lengths.numpy())
    assert h2d == _expected_h2d(b, b.lengths.numpy(), True) - B * (K1 - 1) * 4 + B * 4
