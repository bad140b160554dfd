"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function that ``include/sv.h`` declares, sizes its workspace, and
rejects bad arguments synchronously, before any CUDA call."""
import ctypes
import os
import re

import pytest

import speculative_decoding_verification_93_b200 as sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sv_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = sv.lib()
    names = declared_functions()
    assert "sv_verify" in names and "sv_schedule" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version():
    assert sv.sv_status_string(0) == "SV_OK"
    assert sv.sv_status_string(4) == "SV_ERR_WORKSPACE"
    assert sv.sv_status_string(99) == "SV_UNKNOWN"
    assert sv.lib().sv_version() >= 1
    assert sv.sv_verify_launches() == 3


def test_workspace_bytes():
    n = sv.sv_verify_workspace_bytes(256, 8, 129280, sv.SV_BF16)
    # counters + row counters + row offsets + partials (B * (2K+1) * C float4)
    assert n >= 256 * 17 * 4 * 16
    assert n < 4 * 1024 * 1024
    assert sv.sv_verify_workspace_bytes(0, 8, 100, sv.SV_F32) == 0
    assert sv.sv_verify_workspace_bytes(4, 0, 100, sv.SV_F32) == 0
    assert sv.sv_verify_workspace_bytes(4, 65, 100, sv.SV_F32) == 0
    assert sv.sv_verify_workspace_bytes(4, 4, 0, sv.SV_F32) == 0
    assert sv.sv_verify_workspace_bytes(4, 4, 100, 7) == 0
    # fp32 needs twice the chunks of bf16 at the same V
    a = sv.sv_verify_workspace_bytes(64, 4, 129280, sv.SV_F32)
    b = sv.sv_verify_workspace_bytes(64, 4, 129280, sv.SV_BF16)
    assert a > b


def _call_verify(**kw):
    L = sv.lib()
    args = dict(zt=1 << 20, zd=1 << 21, dtype=sv.SV_BF16, B=4, K=4, V=1000, tok=1 << 22,
                ln=1 << 23, temp=1 << 24, seed=0, row_base=0, ot=1 << 25, oa=1 << 26,
                ws=1 << 27, wsb=1 << 30, status=None, stream=None)
    args.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return L.sv_verify(v(args["zt"]), v(args["zd"]), args["dtype"], args["B"], args["K"],
                       args["V"], v(args["tok"]), v(args["ln"]), v(args["temp"]),
                       ctypes.c_uint64(args["seed"]), args["row_base"], v(args["ot"]),
                       v(args["oa"]), v(args["ws"]), args["wsb"], v(args["status"]),
                       v(args["stream"]))


@pytest.mark.parametrize("kw,code", [
    (dict(zt=None), 1), (dict(tok=None), 1), (dict(ln=None), 1), (dict(temp=None), 1),
    (dict(ot=None), 1), (dict(oa=None), 1), (dict(ws=None), 1),
    (dict(dtype=5), 3), (dict(B=0), 2), (dict(K=0), 2), (dict(K=65), 2), (dict(V=0), 2),
    (dict(row_base=-1), 1), (dict(zt=(1 << 20) + 1), 1), (dict(ws=(1 << 27) + 8), 1),
    (dict(wsb=16), 4),
])
def test_verify_rejects_bad_arguments_on_host(kw, code):
    assert _call_verify(**kw) == code


def test_schedule_and_philox_reject_bad_arguments_on_host():
    L = sv.lib()
    p = ctypes.c_void_p(1 << 20)
    assert L.sv_schedule(None, 4, 4, ctypes.c_float(0.3), p, None) == 1
    assert L.sv_schedule(p, 0, 4, ctypes.c_float(0.3), p, None) == 2
    assert L.sv_schedule(p, 4, 65, ctypes.c_float(0.3), p, None) == 2
    assert L.sv_philox_uniforms(ctypes.c_uint64(0), None, p, p, 4, p, None) == 1
    assert L.sv_philox_uniforms(ctypes.c_uint64(0), p, p, p, -1, p, None) == 2
    assert L.sv_philox_uniforms(ctypes.c_uint64(0), None, None, None, 0, None, None) == 0
    assert L.sv_philox4x32_10(None, p, 3, p, None) == 1
    assert L.sv_verify_debug(p, p, 1, 4, 4, 10, p, p, p, ctypes.c_uint64(0), 0, p, p, p,
                             1 << 20, None, None, None) == 1


def test_python_binding_marshals_only():
    import torch
    zt = torch.zeros(2, 3, 5)
    with pytest.raises(TypeError):
        sv.sv_verify(zt.double(), None, torch.zeros(2, 2, dtype=torch.int32),
                     torch.zeros(2, dtype=torch.int32), torch.zeros(2), 0, None, None, None)


def test_sts_arguments_rejected_on_host():
    L = sv.lib()
    v = ctypes.c_void_p
    big = 1 << 30
    ok = dict(l=1 << 20, a=1 << 21, N=100, K=4, tmin=0.01, tmax=100.0, T=1 << 22, ws=1 << 23,
              wsb=big)

    def call(**kw):
        d = dict(ok)
        d.update(kw)
        return L.sv_sts_fit(v(d["l"]) if d["l"] else None, v(d["a"]) if d["a"] else None,
                            d["N"], d["K"], ctypes.c_float(d["tmin"]), ctypes.c_float(d["tmax"]),
                            v(d["T"]) if d["T"] else None, None, v(d["ws"]) if d["ws"] else None,
                            d["wsb"], None)
    assert call(l=0) == 1 and call(a=0) == 1 and call(T=0) == 1 and call(ws=0) == 1
    assert call(tmin=0.0) == 1 and call(tmax=0.005) == 1 and call(tmax=float("inf")) == 1
    assert call(K=65) == 2 and call(K=0) == 2 and call(N=0) == 2
    assert call(wsb=16) == 4
    assert call(ws=(1 << 23) + 4) == 1
    assert sv.sv_sts_workspace_bytes(100, 4) > 0 and sv.sv_sts_workspace_bytes(100, 65) == 0
    assert L.sv_sts_apply(None, v(1), 1, 1, v(1), None) == 1
    assert L.sv_sts_apply(v(1), v(1), 1, 65, v(1), None) == 2


def test_vocab_parallel_arguments_rejected_on_host():
    L = sv.lib()
    v = ctypes.c_void_p
    big = 1 << 30

    def sl(**kw):
        d = dict(t=1 << 20, d=1 << 21, dtype=sv.SV_BF16, B=4, K=4, V=1000, v0=0, Vs=500, n=2, r=0)
        d.update(kw)
        return sv.sv_vp_slice(d["t"], d["d"], d["dtype"], d["B"], d["K"], d["V"], d["v0"],
                              d["Vs"], d["n"], d["r"])
    ok = sl()
    assert sv.sv_vp_stats_bytes(ok) == 4 * 9 * 1 * 16
    assert sv.sv_vp_workspace_bytes(ok) > 0
    # largest slice sets the chunk count on every rank: 129280 bf16 / 1 rank
    assert sv.sv_vp_stats_bytes(sl(V=129280, Vs=129280, n=1)) == 4 * 9 * 4 * 16
    for bad in (sl(Vs=501), sl(v0=501), sl(r=2), sl(n=1001, Vs=1), sl(K=65), sl(K=0), sl(B=0),
                sl(V=0), sl(dtype=7), sl(Vs=0), sl(v0=-1), sl(V=(1 << 20) + 1)):
        assert sv.sv_vp_stats_bytes(bad) == 0 and sv.sv_vp_workspace_bytes(bad) == 0
    p = v(1 << 22)
    R = ctypes.byref
    assert L.sv_vp_stats(None, p, p, p, p, None) == 1
    assert L.sv_vp_stats(R(sl(t=0)), p, p, p, p, None) == 1
    assert L.sv_vp_stats(R(ok), None, p, p, p, None) == 1
    assert L.sv_vp_stats(R(ok), p, p, p, v((1 << 22) + 8), None) == 1
    assert L.sv_vp_stats(R(sl(dtype=5)), p, p, p, p, None) == 3
    assert L.sv_vp_stats(R(sl(Vs=600)), p, p, p, p, None) == 2
    assert L.sv_vp_stats(R(sl(t=(1 << 20) + 1)), p, p, p, p, None) == 1

    def decide(s=ok, stats=p, ws=p, wsb=big, row_base=0, mass=p):
        return L.sv_vp_decide(R(s), stats, p, p, p, ctypes.c_uint64(0), row_base, p, p, mass,
                              None, ws, wsb, None, None)
    assert decide(wsb=16) == 4
    assert decide(row_base=-1) == 1
    assert decide(stats=v((1 << 22) + 4)) == 1
    assert decide(ws=v((1 << 22) + 8)) == 1
    assert decide(mass=v((1 << 22) + 4)) == 1
    assert decide(stats=None) == 1
    assert decide(s=sl(K=65)) == 2
    assert L.sv_vp_draw(R(ok), p, p, p, 16, None, None) == 4
    assert L.sv_vp_draw(R(ok), v((1 << 22) + 4), p, p, big, None, None) == 1
    assert L.sv_vp_draw(R(ok), None, p, p, big, None, None) == 1
    assert L.sv_vp_draw(R(sl(r=-1)), p, p, p, big, None, None) == 2


def test_verify_host_arguments_rejected_on_host():
    L = sv.lib()
    v = ctypes.c_void_p
    n = sv.sv_verify_host_workspace_bytes(4, 4, 1000, sv.SV_BF16)
    assert n > 4 * 5 * 1000 * 2 + 4 * 4 * 1000 * 2
    assert sv.sv_verify_host_workspace_bytes(4, 65, 1000, sv.SV_BF16) == 0
    assert sv.sv_verify_host_workspace_bytes(4, 4, 1000, 9) == 0
    p = v(1 << 20)
    ws = v(1 << 24)

    def call(zt=p, conf=p, tok=p, temp=p, ot=p, oa=p, ln=p, w=ws, wsb=1 << 40, dtype=sv.SV_BF16,
             B=4, K=4, V=1000, row_base=0):
        return L.sv_verify_host(zt, None, dtype, B, K, V, conf, ctypes.c_float(0.3), tok, temp,
                                ctypes.c_uint64(0), row_base, ot, oa, ln, None, 1, w, wsb, None,
                                None)
    for kw in ("zt", "tok", "temp", "ot", "oa", "ln", "w"):
        assert call(**{kw: None}) == 1, kw
    assert call(dtype=4) == 3
    assert call(K=0) == 2 and call(B=0) == 2 and call(V=(1 << 20) + 1) == 2
    assert call(row_base=-1) == 1
    assert call(w=v((1 << 24) + 16)) == 1
    assert call(wsb=n - 1) == 4


def _declared_arity():
    """Parameter count of every function declared in include/sv.h."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    out = {}
    for m in re.finditer(r"\b(sv_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_header():
    L = sv.lib()
    arity = _declared_arity()
    assert "sv_verify_host" in arity and "sv_vp_decide" in arity
    checked = 0
    for name, n in arity.items():
        fn = getattr(L, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
            checked += 1
    assert checked >= 20


def test_schedule_verify_arguments_rejected_on_host():
    L = sv.lib()
    v = ctypes.c_void_p
    p = v(1 << 20)
    ws = v(1 << 24)
    n = sv.sv_verify_workspace_bytes(4, 4, 1000, sv.SV_BF16)

    def call(zt=p, tok=p, conf=p, ln=p, temp=p, ot=p, oa=p, w=ws, wsb=1 << 40, dtype=sv.SV_BF16,
             B=4, K=4, V=1000, row_base=0):
        return L.sv_schedule_verify(zt, None, dtype, B, K, V, tok, conf, ctypes.c_float(0.3), ln,
                                    temp, ctypes.c_uint64(0), row_base, ot, oa, w, wsb, None, None)
    for kw in ("zt", "tok", "conf", "ln", "temp", "ot", "oa", "w"):
        assert call(**{kw: None}) == 1, kw
    assert call(dtype=4) == 3
    assert call(K=0) == 2 and call(B=0) == 2 and call(V=(1 << 20) + 1) == 2
    assert call(row_base=-1) == 1
    assert call(w=v((1 << 24) + 8)) == 1
    assert call(wsb=n - 1) == 4
