"""The allocation-free entry point, sv_verify_noalloc, for callers that may
not allocate device memory while they verify (a serving loop that plans its
memory up front, a plain C host program with no device allocator).  It must
give exactly what sv_verify gives with a caller-owned workspace, call after
call, although every call reuses the library's one fixed scratch array.

Kept in a file of its own that pytest collects last, so that a run stopping
at the first failure has already run every other test; it also passes alone
in a fresh process."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_93_b200 as sv
from speculative_decoding_verification_93_b200 import workloads

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _with_workspace(b, seed, row_base=0):
    B, K1, V = b.zt.shape
    dt = sv.SV_BF16 if b.zt.dtype == torch.bfloat16 else sv.SV_F32
    ws = torch.empty(sv.sv_verify_workspace_bytes(B, K1 - 1, V, dt), dtype=torch.uint8,
                     device="cuda")
    tok = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sv.sv_verify(b.zt, b.zd, b.tokens, b.lengths, b.temperature, seed, tok, acc, ws, status=st,
                 row_base=row_base)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), acc.cpu().numpy(), int(st.item())


def _no_alloc(b, seed, row_base=0):
    B, K1, V = b.zt.shape
    tok = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sv.sv_verify_noalloc(b.zt, b.zd, b.tokens, b.lengths, b.temperature, seed, tok, acc,
                         status=st, row_base=row_base)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), acc.cpu().numpy(), int(st.item())


def _cuda(b):
    for n in ("zt", "zd", "tokens", "temperature", "conf", "lengths"):
        setattr(b, n, getattr(b, n).cuda())
    return b


@pytest.mark.parametrize("name", ["c1", "c3"])
def test_no_alloc_matches_sv_verify_on_consecutive_calls(name):
    b = workloads.make_batch(name, device="cuda")
    B, K1, V = b.zt.shape
    dt = sv.SV_BF16 if b.zt.dtype == torch.bfloat16 else sv.SV_F32
    assert sv.sv_verify_workspace_bytes(B, K1 - 1, V, dt) <= SCRATCH_BYTES
    for call, seed in enumerate((101, 202)):
        want = _with_workspace(b, seed)
        got = _no_alloc(b, seed)
        np.testing.assert_array_equal(got[0], want[0], err_msg=f"call {call}: tokens")
        np.testing.assert_array_equal(got[1], want[1], err_msg=f"call {call}: accept lengths")
        assert got[2] == want[2] == 0


def test_no_alloc_back_to_back_shapes_and_row_base():
    """Consecutive calls with different shapes, dtypes and row bases leave no
    state behind that changes the next call's result."""
    cases = [workloads.random_small(48, 5, 40000, dtype=torch.bfloat16, seed=3,
                                    temps=(0.0, 0.7, 1.0)),
             workloads.random_small(16, 3, 1001, dtype=torch.float32, seed=4),
             workloads.random_small(48, 5, 40000, dtype=torch.bfloat16, seed=3,
                                    temps=(0.0, 0.7, 1.0))]
    for i, b in enumerate(cases):
        b = _cuda(b)
        want = _with_workspace(b, 9 + i, row_base=1000 * i)
        got = _no_alloc(b, 9 + i, row_base=1000 * i)
        np.testing.assert_array_equal(got[0], want[0])
        np.testing.assert_array_equal(got[1], want[1])


def test_no_alloc_rejects_batches_beyond_its_scratch():
    B, K, V = 8192, 64, 129280         # fp32: needs more than 16 MiB of scratch
    need = sv.sv_verify_workspace_bytes(B, K, V, sv.SV_F32)
    assert need > SCRATCH_BYTES
    zt = torch.zeros(1, dtype=torch.float32, device="cuda")
    ptr = torch.zeros(B * (K + 1) + 16, dtype=torch.int32, device="cuda")
    L = sv.lib()
    import ctypes
    p = ctypes.c_void_p
    rc = L.sv_verify_noalloc(p(zt.data_ptr()), p(zt.data_ptr()), sv.SV_F32, B, K, V,
                             p(ptr.data_ptr()), p(ptr.data_ptr()), p(zt.data_ptr()),
                             ctypes.c_uint64(0), 0, p(ptr.data_ptr()), p(ptr.data_ptr()), None,
                             None)
    assert rc == 4 and sv.sv_status_string(rc) == "SV_ERR_WORKSPACE"
