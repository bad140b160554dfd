"""sv_schedule_verify: the schedule computed inside the verification prologue.
Its lengths and outputs must equal, bit for bit, sv_schedule followed by
sv_verify on the same inputs -- both take the lengths from the same device
function -- including rows the verification marks invalid, thresholds that
keep every draft or none, NaN confidences, and the full c2 workload."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200 import workloads
from _parity import gpu_schedule, gpu_verify

pytestmark = pytest.mark.gpu


def fused(zt, zd, tokens, conf, tau, temperature, seed, row_base=0):
    B, K1, V = zt.shape
    K = K1 - 1
    dt = sv.SV_BF16 if zt.dtype == torch.bfloat16 else sv.SV_F32
    ws = torch.randint(0, 255, (sv.sv_verify_workspace_bytes(B, K, V, dt),), dtype=torch.uint8,
                       device=zt.device)
    ln = torch.full((B,), -7, dtype=torch.int32, device=zt.device)
    ot = torch.full((B, K1), -7, dtype=torch.int32, device=zt.device)
    oa = torch.full((B,), -7, dtype=torch.int32, device=zt.device)
    st = torch.zeros(1, dtype=torch.int32, device=zt.device)
    sv.sv_schedule_verify(zt, zd, tokens, conf, tau, ln, temperature, seed, ot, oa, ws, status=st,
                          row_base=row_base)
    torch.cuda.synchronize()
    return ln.cpu().numpy(), ot.cpu().numpy(), oa.cpu().numpy(), int(st.item())


def two_calls(zt, zd, tokens, conf, tau, temperature, seed, row_base=0):
    ln = gpu_schedule(conf, tau)
    g = gpu_verify(zt, zd, tokens, ln, temperature, seed, row_base=row_base)
    return ln.cpu().numpy(), g["tokens"], g["accept"], g["status"]


def assert_same(a, b):
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)
    assert a[3] == b[3]


@pytest.mark.parametrize("V,dtype,K,B", [(1000, torch.float32, 4, 33), (1001, torch.bfloat16, 8, 64),
                                         (65543, torch.bfloat16, 3, 16)])
@pytest.mark.parametrize("tau", [-1.0, 0.0, 0.3, 0.9, 1.5, float("nan")])
def test_equals_schedule_then_verify(V, dtype, K, B, tau):
    b = workloads.random_small(B, K, V, dtype=dtype, seed=V + K, temps=(0.0, 0.6, 1.0),
                               device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(K)
    conf = torch.rand(B, K, generator=g, device="cuda") ** 0.3
    conf[0, 1] = float("nan")   # counts as 0: the row keeps at most one draft
    conf[1] = 1.0
    for zd in (b.zd, None):
        assert_same(fused(b.zt, zd, b.tokens, conf, tau, b.temperature, 5, row_base=3),
                    two_calls(b.zt, zd, b.tokens, conf, tau, b.temperature, 5, row_base=3))


def test_invalid_rows():
    B, K, V = 12, 4, 1000
    b = workloads.random_small(B, K, V, seed=1, temps=(0.0, 1.0), device="cuda")
    conf = torch.full((B, K), 0.99, device="cuda")
    tokens = b.tokens.clone()
    tokens[2, 0] = V                 # out of range, inside the scheduled prefix
    tokens[3, K - 1] = -5            # out of range, scheduled too (tau keeps all)
    temp = b.temperature.clone()
    temp[4] = float("inf")
    temp[5] = -1.0
    a = fused(b.zt, b.zd, tokens, conf, 0.5, temp, 9)
    assert_same(a, two_calls(b.zt, b.zd, tokens, conf, 0.5, temp, 9))
    assert a[2][2] == -1 and a[2][3] == -1 and a[2][4] == -1 and a[2][5] == -1
    assert a[3] & sv.SV_ROW_BAD_TOKEN and a[3] & sv.SV_ROW_BAD_TEMPERATURE


def test_full_c2():
    bt = workloads.make_batch("c2", device="cuda")
    for seed in (0, 1):
        assert_same(fused(bt.zt, bt.zd, bt.tokens, bt.conf, bt.tau, bt.temperature, seed),
                    two_calls(bt.zt, bt.zd, bt.tokens, bt.conf, bt.tau, bt.temperature, seed))
