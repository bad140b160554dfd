"""ctypes binding of the C ABI in ``include/sv.h`` (same names, same
arguments).  Tensors are passed by device pointer; the stream defaults to
PyTorch's current stream on the tensors' device."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

SV_F32, SV_BF16 = 0, 1
SV_ROW_BAD_TOKEN, SV_ROW_BAD_LENGTH, SV_ROW_BAD_TEMPERATURE = 1, 2, 4
SV_NOTE_ZERO_RESIDUAL, SV_NOTE_CDF_FALLBACK = 8, 16
_STATUS = {0: "SV_OK", 1: "SV_ERR_ARG", 2: "SV_ERR_SHAPE", 3: "SV_ERR_DTYPE",
           4: "SV_ERR_WORKSPACE", 5: "SV_ERR_CUDA"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsv.so")
_lib = None


class SVError(RuntimeError):
    def __init__(self, fn: str, code: int):
        extra = ""
        if code == 5 and _lib is not None:
            extra = f" (cuda error {_lib.sv_last_cuda_error()})"
        super().__init__(f"{fn} failed: {_STATUS.get(code, code)}{extra}")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load ``libsv.so``; raises if it is missing (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m speculative_decoding_verification_93_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, u64, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                             ctypes.c_size_t)
    L.sv_schedule.argtypes = [vp, i32, i32, ctypes.c_float, vp, vp]
    L.sv_schedule_admit.argtypes = [vp, i32, i32, vp, i32, vp, vp, vp]
    L.sv_sts_workspace_bytes.argtypes = [i32, i32]
    L.sv_sts_workspace_bytes.restype = sz
    L.sv_sts_fit.argtypes = [vp, vp, i32, i32, ctypes.c_float, ctypes.c_float, vp, vp, vp, sz,
                             vp]
    L.sv_sts_apply.argtypes = [vp, vp, i32, i32, vp, vp]
    L.sv_debug_sts_wait_limit.argtypes = [u64]
    L.sv_debug_sts_wait_limit.restype = i32
    L.sv_debug_sts_timeouts.argtypes = []
    L.sv_debug_sts_timeouts.restype = i32
    L.sv_verify_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.sv_verify_workspace_bytes.restype = sz
    L.sv_verify.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, u64, i64, vp, vp, vp, sz, vp,
                            vp]
    L.sv_schedule_verify.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, ctypes.c_float, vp, vp,
                                     u64, i64, vp, vp, vp, sz, vp, vp]
    L.sv_verify_debug.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, u64, i64, vp, vp, vp,
                                  sz, vp, vp, vp]
    L.sv_verify_noalloc.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, u64, i64, vp, vp, vp,
                                    vp]
    sp = ctypes.POINTER(sv_vp_slice)
    L.sv_vp_stats_bytes.argtypes = [sp]
    L.sv_vp_stats_bytes.restype = sz
    L.sv_vp_workspace_bytes.argtypes = [sp]
    L.sv_vp_workspace_bytes.restype = sz
    L.sv_vp_stats.argtypes = [sp, vp, vp, vp, vp, vp]
    L.sv_vp_decide.argtypes = [sp, vp, vp, vp, vp, u64, i64, vp, vp, vp, vp, vp, sz, vp, vp]
    L.sv_vp_draw.argtypes = [sp, vp, vp, vp, sz, vp, vp]
    L.sv_verify_host_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.sv_verify_host_workspace_bytes.restype = sz
    L.sv_verify_host.argtypes = [vp, vp, i32, i32, i32, i32, vp, ctypes.c_float, vp, vp, u64, i64,
                                 vp, vp, vp, vp, i32, vp, sz, vp, vp]
    L.sv_philox_uniforms.argtypes = [u64, vp, vp, vp, i32, vp, vp]
    L.sv_philox4x32_10.argtypes = [vp, vp, i32, vp, vp]
    L.sv_profile_begin.argtypes = [i32]
    L.sv_profile_read.argtypes = [vp, i32]
    L.sv_profile_read.restype = i32
    L.sv_status_string.argtypes = [i32]
    L.sv_status_string.restype = ctypes.c_char_p
    for name in ("sv_schedule", "sv_schedule_admit", "sv_sts_fit", "sv_sts_apply", "sv_verify",
                 "sv_verify_debug", "sv_verify_noalloc", "sv_verify_host", "sv_vp_stats",
                 "sv_vp_decide",
                 "sv_vp_draw",
                 "sv_philox_uniforms",
                 "sv_philox4x32_10", "sv_profile_begin"):
        getattr(L, name).restype = i32
    L.sv_last_cuda_error.restype = i32
    L.sv_version.restype = i32
    L.sv_verify_launches.restype = i32
    _lib = L
    return L


class sv_vp_slice(ctypes.Structure):
    """This rank's slice of the vocabulary (``sv_vp_slice`` in include/sv.h)."""
    _fields_ = [("target_logits", ctypes.c_void_p), ("draft_logits", ctypes.c_void_p),
                ("dtype", ctypes.c_int), ("B", ctypes.c_int), ("K", ctypes.c_int),
                ("V", ctypes.c_int), ("v0", ctypes.c_int), ("Vs", ctypes.c_int),
                ("nshards", ctypes.c_int), ("shard", ctypes.c_int)]


def vp_slice(target_logits, draft_logits, V: int, v0: int, nshards: int,
             shard: int) -> sv_vp_slice:
    """Describe a slice from its logits: target [B, K+1, Vs], draft [B, K, Vs]
    or None, holding tokens v0 .. v0+Vs-1 of a vocabulary of V."""
    B, K1, Vs = target_logits.shape
    dt = _dtype(target_logits)
    if not target_logits.is_contiguous():
        raise TypeError("target_logits must be contiguous")
    if draft_logits is not None and (draft_logits.dtype != target_logits.dtype
                                     or not draft_logits.is_contiguous()
                                     or tuple(draft_logits.shape) != (B, K1 - 1, Vs)):
        raise TypeError("draft_logits must be a contiguous [B, K, Vs] tensor of the target dtype")
    return sv_vp_slice(target_logits.data_ptr(),
                       None if draft_logits is None else draft_logits.data_ptr(),
                       dt, B, K1 - 1, int(V), int(v0), Vs, int(nshards), int(shard))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, like: torch.Tensor):
    if stream is None:
        stream = torch.cuda.current_stream(like.device)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn: str, code: int):
    if code != 0:
        raise SVError(fn, code)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SV_F32
    if t.dtype == torch.bfloat16:
        return SV_BF16
    raise TypeError(f"logits must be float32 or bfloat16, got {t.dtype}")


def _need(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {dtype} tensor")


def sv_schedule(conf: torch.Tensor, load: float, lengths: torch.Tensor, stream=None) -> None:
    _need(conf, torch.float32, "conf")
    _need(lengths, torch.int32, "lengths")
    B, K = conf.shape
    _check("sv_schedule", lib().sv_schedule(_ptr(conf), B, K, float(load), _ptr(lengths),
                                            _stream(stream, conf)))


def sv_schedule_admit(conf: torch.Tensor, speed: torch.Tensor, lengths: torch.Tensor,
                      tau_out: Optional[torch.Tensor] = None, stream=None) -> None:
    _need(conf, torch.float32, "conf")
    _need(speed, torch.float32, "speed")
    _need(lengths, torch.int32, "lengths")
    B, K = conf.shape
    _check("sv_schedule_admit", lib().sv_schedule_admit(
        _ptr(conf), B, K, _ptr(speed), speed.numel(), _ptr(lengths), _ptr(tau_out),
        _stream(stream, conf)))


def sv_sts_workspace_bytes(N: int, K: int) -> int:
    return int(lib().sv_sts_workspace_bytes(N, K))


def sv_sts_fit(logits: torch.Tensor, accept_len: torch.Tensor, temperature: torch.Tensor,
               ece: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               tmin: float = 1e-2, tmax: float = 1e2, stream=None) -> None:
    _need(logits, torch.float32, "logits")
    _need(accept_len, torch.int32, "accept_len")
    _need(temperature, torch.float32, "temperature")
    N, K = logits.shape
    if workspace is None:
        workspace = torch.empty(sv_sts_workspace_bytes(N, K), dtype=torch.uint8,
                                device=logits.device)
    _check("sv_sts_fit", lib().sv_sts_fit(
        _ptr(logits), _ptr(accept_len), N, K, float(tmin), float(tmax), _ptr(temperature),
        _ptr(ece), _ptr(workspace), workspace.numel(), _stream(stream, logits)))


def sv_sts_apply(logits: torch.Tensor, temperature: torch.Tensor, conf_out: torch.Tensor,
                 stream=None) -> None:
    _need(logits, torch.float32, "logits")
    _need(temperature, torch.float32, "temperature")
    _need(conf_out, torch.float32, "conf_out")
    N, K = logits.shape
    _check("sv_sts_apply", lib().sv_sts_apply(_ptr(logits), _ptr(temperature), N, K,
                                              _ptr(conf_out), _stream(stream, logits)))


def sv_debug_sts_wait_limit(limit_ns: int) -> None:
    """Test export: wall-time limit of the calibration barrier's wait on the
    current device (0 restores the 1 s default)."""
    _check("sv_debug_sts_wait_limit", lib().sv_debug_sts_wait_limit(int(limit_ns)))


def sv_debug_sts_timeouts() -> int:
    """Test export: barrier waits that ran out since the previous call."""
    n = lib().sv_debug_sts_timeouts()
    if n < 0:
        raise SVError("sv_debug_sts_timeouts", 5)
    return n


def sv_verify_workspace_bytes(B: int, K: int, V: int, dtype: int) -> int:
    return int(lib().sv_verify_workspace_bytes(B, K, V, dtype))


def _verify_args(target_logits, draft_logits, draft_tokens, lengths, temperature):
    B, K1, V = target_logits.shape
    K = K1 - 1
    dt = _dtype(target_logits)
    if not target_logits.is_contiguous():
        raise TypeError("target_logits must be contiguous")
    if draft_logits is not None and (draft_logits.dtype != target_logits.dtype
                                     or not draft_logits.is_contiguous()
                                     or tuple(draft_logits.shape) != (B, K, V)):
        raise TypeError("draft_logits must be a contiguous [B, K, V] tensor of the target dtype")
    _need(draft_tokens, torch.int32, "draft_tokens")
    _need(lengths, torch.int32, "lengths")
    _need(temperature, torch.float32, "temperature")
    return B, K, V, dt


def sv_verify(target_logits, draft_logits, draft_tokens, lengths, temperature, seed: int,
              out_tokens, out_accept_len, workspace, status=None, row_base: int = 0,
              stream=None) -> None:
    B, K, V, dt = _verify_args(target_logits, draft_logits, draft_tokens, lengths, temperature)
    _check("sv_verify", lib().sv_verify(
        _ptr(target_logits), _ptr(draft_logits), dt, B, K, V, _ptr(draft_tokens), _ptr(lengths),
        _ptr(temperature), ctypes.c_uint64(seed & (2**64 - 1)), int(row_base), _ptr(out_tokens),
        _ptr(out_accept_len), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream, target_logits)))


def sv_schedule_verify(target_logits, draft_logits, draft_tokens, conf, load: float, lengths,
                       temperature, seed: int, out_tokens, out_accept_len, workspace, status=None,
                       row_base: int = 0, stream=None) -> None:
    """sv_schedule then sv_verify in one call: `lengths` receives the
    scheduled lengths (see include/sv.h)."""
    B, K, V, dt = _verify_args(target_logits, draft_logits, draft_tokens, lengths, temperature)
    _need(conf, torch.float32, "conf")
    if tuple(conf.shape) != (B, K):
        raise TypeError("conf must be a [B, K] float32 tensor")
    _check("sv_schedule_verify", lib().sv_schedule_verify(
        _ptr(target_logits), _ptr(draft_logits), dt, B, K, V, _ptr(draft_tokens), _ptr(conf),
        float(load), _ptr(lengths), _ptr(temperature), ctypes.c_uint64(seed & (2**64 - 1)),
        int(row_base), _ptr(out_tokens), _ptr(out_accept_len), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream, target_logits)))


def sv_verify_debug(target_logits, draft_logits, draft_tokens, lengths, temperature, seed: int,
                    out_tokens, out_accept_len, workspace, stats_out, status=None,
                    row_base: int = 0, stream=None) -> None:
    B, K, V, dt = _verify_args(target_logits, draft_logits, draft_tokens, lengths, temperature)
    _check("sv_verify_debug", lib().sv_verify_debug(
        _ptr(target_logits), _ptr(draft_logits), dt, B, K, V, _ptr(draft_tokens), _ptr(lengths),
        _ptr(temperature), ctypes.c_uint64(seed & (2**64 - 1)), int(row_base), _ptr(out_tokens),
        _ptr(out_accept_len), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _ptr(stats_out), _stream(stream, target_logits)))


def sv_verify_noalloc(target_logits, draft_logits, draft_tokens, lengths, temperature, seed: int,
                      out_tokens, out_accept_len, status=None, row_base: int = 0,
                      stream=None) -> None:
    """sv_verify with the library's own fixed scratch instead of a workspace,
    for callers that must not allocate device memory (see include/sv.h)."""
    B, K, V, dt = _verify_args(target_logits, draft_logits, draft_tokens, lengths, temperature)
    _check("sv_verify_noalloc", lib().sv_verify_noalloc(
        _ptr(target_logits), _ptr(draft_logits), dt, B, K, V, _ptr(draft_tokens), _ptr(lengths),
        _ptr(temperature), ctypes.c_uint64(seed & (2**64 - 1)), int(row_base), _ptr(out_tokens),
        _ptr(out_accept_len), _ptr(status), _stream(stream, target_logits)))


def sv_vp_stats_bytes(slice_: sv_vp_slice) -> int:
    return int(lib().sv_vp_stats_bytes(ctypes.byref(slice_)))


def sv_vp_workspace_bytes(slice_: sv_vp_slice) -> int:
    return int(lib().sv_vp_workspace_bytes(ctypes.byref(slice_)))


def sv_vp_stats(slice_: sv_vp_slice, draft_tokens, lengths, temperature, stats_local,
                stream=None) -> None:
    _need(draft_tokens, torch.int32, "draft_tokens")
    _need(lengths, torch.int32, "lengths")
    _need(temperature, torch.float32, "temperature")
    _check("sv_vp_stats", lib().sv_vp_stats(
        ctypes.byref(slice_), _ptr(draft_tokens), _ptr(lengths), _ptr(temperature),
        _ptr(stats_local), _stream(stream, lengths)))


def sv_vp_decide(slice_: sv_vp_slice, stats_all, draft_tokens, lengths, temperature, seed: int,
                 out_tokens, out_accept_len, mass_local, workspace, status=None, norm_out=None,
                 row_base: int = 0, stream=None) -> None:
    _need(draft_tokens, torch.int32, "draft_tokens")
    _need(lengths, torch.int32, "lengths")
    _need(temperature, torch.float32, "temperature")
    _check("sv_vp_decide", lib().sv_vp_decide(
        ctypes.byref(slice_), _ptr(stats_all), _ptr(draft_tokens), _ptr(lengths),
        _ptr(temperature), ctypes.c_uint64(seed & (2**64 - 1)), int(row_base), _ptr(out_tokens),
        _ptr(out_accept_len), _ptr(mass_local), _ptr(norm_out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream, lengths)))


def sv_vp_draw(slice_: sv_vp_slice, mass_all, out_tokens, workspace, status=None,
               stream=None) -> None:
    _check("sv_vp_draw", lib().sv_vp_draw(
        ctypes.byref(slice_), _ptr(mass_all), _ptr(out_tokens), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream, out_tokens)))


def sv_verify_host_workspace_bytes(B: int, K: int, V: int, dtype: int) -> int:
    return int(lib().sv_verify_host_workspace_bytes(B, K, V, dtype))


def _need_host(t: torch.Tensor, dtype, name: str):
    if t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {dtype} host tensor")


def sv_verify_host(target_logits, draft_logits, conf, load: float, draft_tokens, temperature,
                   seed: int, out_tokens, out_accept_len, lengths, workspace, status=None,
                   row_base: int = 0, levelwise: bool = False, stream=None) -> int:
    """Host-resident inputs and outputs (pinned CPU tensors), device
    workspace; returns the bytes copied host-to-device.  With conf None,
    `lengths` is an input and no schedule runs.  levelwise copies only the
    logits the outcome depends on, one position level at a time.  The
    outputs are valid once `stream` has drained."""
    B, K1, V = target_logits.shape
    K = K1 - 1
    if target_logits.is_cuda or not target_logits.is_contiguous():
        raise TypeError("target_logits must be a contiguous host tensor")
    dt = _dtype(target_logits)
    if draft_logits is not None:
        _need_host(draft_logits, target_logits.dtype, "draft_logits")
        if tuple(draft_logits.shape) != (B, K, V):
            raise TypeError("draft_logits must be [B, K, V]")
    if conf is not None:
        _need_host(conf, torch.float32, "conf")
    _need_host(draft_tokens, torch.int32, "draft_tokens")
    _need_host(temperature, torch.float32, "temperature")
    _need_host(out_tokens, torch.int32, "out_tokens")
    _need_host(out_accept_len, torch.int32, "out_accept_len")
    _need_host(lengths, torch.int32, "lengths")
    if status is not None:
        _need_host(status, torch.int32, "status")
    if not workspace.is_cuda:
        raise TypeError("workspace must be device memory")
    h2d = ctypes.c_size_t(0)
    _check("sv_verify_host", lib().sv_verify_host(
        _ptr(target_logits), _ptr(draft_logits), dt, B, K, V, _ptr(conf), float(load),
        _ptr(draft_tokens), _ptr(temperature), ctypes.c_uint64(seed & (2**64 - 1)), int(row_base),
        _ptr(out_tokens), _ptr(out_accept_len), _ptr(lengths), _ptr(status),
        1 if levelwise else 0, _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(h2d),
        _stream(stream, workspace)))
    return int(h2d.value)


def sv_philox_uniforms(seed: int, row, pos, draw, out, stream=None) -> None:
    n = out.numel()
    _check("sv_philox_uniforms", lib().sv_philox_uniforms(
        ctypes.c_uint64(seed & (2**64 - 1)), _ptr(row), _ptr(pos), _ptr(draw), n, _ptr(out),
        _stream(stream, out)))


def sv_philox4x32_10(ctr, key, out, stream=None) -> None:
    n = out.numel() // 4
    _check("sv_philox4x32_10", lib().sv_philox4x32_10(_ptr(ctr), _ptr(key), n, _ptr(out),
                                                      _stream(stream, out)))


def sv_profile_begin(capacity: int) -> None:
    _check("sv_profile_begin", lib().sv_profile_begin(int(capacity)))


def sv_profile_read(max_n: int = 4096):
    buf = (ctypes.c_float * max_n)()
    n = lib().sv_profile_read(ctypes.cast(buf, ctypes.c_void_p), max_n)
    return [buf[i] for i in range(n)]


def sv_verify_launches() -> int:
    return int(lib().sv_verify_launches())


def sv_status_string(code: int) -> str:
    return lib().sv_status_string(int(code)).decode()


def verify(target_logits, draft_logits, draft_tokens, lengths, temperature, seed: int,
           row_base: int = 0, workspace=None, status=None, stream=None):
    """Allocate the outputs (and workspace, if not given) with PyTorch and call
    :func:`sv_verify`.  Returns (out_tokens [B, K+1], out_accept_len [B])."""
    B, K1, V = target_logits.shape
    dev = target_logits.device
    out_tokens = torch.empty(B, K1, dtype=torch.int32, device=dev)
    out_acc = torch.empty(B, dtype=torch.int32, device=dev)
    if workspace is None:
        n = sv_verify_workspace_bytes(B, K1 - 1, V, _dtype(target_logits))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    sv_verify(target_logits, draft_logits, draft_tokens, lengths, temperature, seed, out_tokens,
              out_acc, workspace, status=status, row_base=row_base, stream=stream)
    return out_tokens, out_acc
