"""Kimi Delta Attention (KDA) operator for NVIDIA B200 — Python binding of libkda.so.

This module only marshals arguments: every step of the operator runs in the CUDA kernels of
``libkda.so`` behind the C ABI declared in ``include/kda.h``. PyTorch supplies device memory and
the current stream. There is no CPU fallback: without the built library every call raises.

Entry points (same names as the C ABI):
  kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk=64, ...)
      chunkwise prefill -> (o, final_state); ``fusion=`` adds the q/k L2 norm, the decay gate and
      the output epilogue (kda_chunk_fwd_fused)
  kda_chunk_fwd_noalloc(...)  the same prefill on the library's own scratch array
  kda_chunk_bwd(q, k, v, log_alpha, beta, d_o, ...)  gradients of the prefill
  kda_recurrent_step(q, k, v, log_alpha, beta, state, o=None, fusion=None)
      one decode token per sequence, ``state`` updated in place -> o
  kda_recurrent_fwd(q, k, v, log_alpha, beta, state_pool, state_indices=None, ...)
      a few tokens per sequence against pooled states -> o
  kda_chunk_fwd_workspace_size(...), kda_chunk_bwd_workspace_size(...), kda_last_device_error(),
  kda_status_string(code), kda_profile_enable(), kda_profile_read()

Every tensor must be contiguous and on the device of q; caller-provided outputs and workspaces are
checked for device, dtype and shape (size) before anything is launched.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import roofline  # noqa: F401  (work counts used by the benchmark)

_PKG = os.path.dirname(os.path.abspath(__file__))
# KDA_LIBRARY selects another build of the library (e.g. the bounds-checked libkda_checked.so)
LIB_PATH = os.environ.get("KDA_LIBRARY") or os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED = 0, 1, 2
KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_WORKSPACE = 3, 4, 5
KDA_DTYPE_F32, KDA_DTYPE_BF16 = 0, 1

# every symbol the headers under include/ declare
ABI_SYMBOLS = ("kda_status_string", "kda_version", "kda_chunk_fwd_workspace_size",
               "kda_chunk_fwd", "kda_recurrent_step", "kda_last_device_error",
               "kda_profile_enable", "kda_profile_read", "kda_chunk_fwd_noalloc",
               "kda_recurrent_fwd", "kda_chunk_fwd_fused", "kda_recurrent_fwd_fused",
               "kda_chunk_bwd_workspace_size", "kda_chunk_bwd", "kda_recurrent_step_fused",
               "kda_selftest_wait_timeout", "kda_selftest_bounds")


class Fusion(ctypes.Structure):
    """kda_fusion_t: in-kernel q/k L2 normalisation, the fused log-space decay gate, and the output
    epilogue (head-wise RMSNorm x sigmoid gate)."""
    _fields_ = [("qk_l2norm", ctypes.c_int32), ("qk_l2norm_eps", ctypes.c_float),
                ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("out_norm", ctypes.c_int32), ("out_norm_eps", ctypes.c_float),
                ("out_norm_weight", ctypes.c_void_p), ("out_gate", ctypes.c_void_p)]


class ProfileEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_double)]

_lock = threading.Lock()
_lib = None


class KDAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {status_string(code)}")


def lib() -> ctypes.CDLL:
    """The loaded libkda.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libkda.so not built at {LIB_PATH}; run "
                                  "`python -m gated_delta_rule_120_b200._build` (or "
                                  "__graft_entry__.build())")
            L = ctypes.CDLL(LIB_PATH)
            vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            L.kda_status_string.argtypes = [ctypes.c_int]
            L.kda_status_string.restype = ctypes.c_char_p
            L.kda_version.argtypes = []
            L.kda_version.restype = ctypes.c_char_p
            L.kda_chunk_fwd_workspace_size.argtypes = [i32] * 7 + [ctypes.c_int,
                                                                   ctypes.POINTER(sz)]
            L.kda_chunk_fwd_workspace_size.restype = ctypes.c_int
            L.kda_chunk_fwd.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i32, i32,
                                        i32, i32, i32, i32, vp, vp, vp, sz, vp]
            L.kda_chunk_fwd.restype = ctypes.c_int
            L.kda_recurrent_step.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i32,
                                             i32, i32, vp]
            L.kda_recurrent_step.restype = ctypes.c_int
            L.kda_recurrent_fwd.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, i32,
                                            i32, i32, i32, i32, i32, vp]
            L.kda_recurrent_fwd.restype = ctypes.c_int
            L.kda_chunk_fwd_fused.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i32,
                                              i32, i32, i32, i32, i32, vp, vp, vp, sz,
                                              ctypes.POINTER(Fusion), vp]
            L.kda_chunk_fwd_fused.restype = ctypes.c_int
            L.kda_recurrent_fwd_fused.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp,
                                                  i32, i32, i32, i32, i32, i32,
                                                  ctypes.POINTER(Fusion), vp]
            L.kda_recurrent_fwd_fused.restype = ctypes.c_int
            L.kda_recurrent_step_fused.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32,
                                                   i32, i32, i32, ctypes.POINTER(Fusion), vp]
            L.kda_recurrent_step_fused.restype = ctypes.c_int
            L.kda_chunk_bwd_workspace_size.argtypes = [i32] * 6 + [ctypes.c_int,
                                                                   ctypes.POINTER(sz)]
            L.kda_chunk_bwd_workspace_size.restype = ctypes.c_int
            L.kda_chunk_bwd.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i32, i32,
                                        i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.kda_chunk_bwd.restype = ctypes.c_int
            L.kda_last_device_error.argtypes = [vp]
            L.kda_last_device_error.restype = ctypes.c_int
            L.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32,
                                                i32, i32, i32, i32, i32, i32, vp, vp, vp]
            L.kda_chunk_fwd_noalloc.restype = ctypes.c_int
            L.kda_profile_enable.argtypes = [ctypes.c_int32]
            L.kda_profile_enable.restype = ctypes.c_int
            L.kda_profile_read.argtypes = [ctypes.POINTER(ProfileEntry), ctypes.c_int32,
                                           ctypes.POINTER(ctypes.c_int32)]
            L.kda_profile_read.restype = ctypes.c_int
            L.kda_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
            L.kda_selftest_wait_timeout.restype = ctypes.c_int
            L.kda_selftest_bounds.argtypes = [vp, sz, vp]
            L.kda_selftest_bounds.restype = ctypes.c_int
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().kda_status_string(int(code)).decode()


kda_status_string = status_string


def _check(code: int, where: str):
    if code != KDA_OK:
        raise KDAError(code, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"q/k/v dtype {t.dtype} not supported (bf16 or fp32)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _on(device: torch.device):
    """Make `device` current around an ABI call: the library launches on (and looks up per-device
    state of) the current device, which must own the tensors and the stream passed to it."""
    return torch.cuda.device(device)


def _need(t: torch.Tensor, name: str, device, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor, got one on {t.device}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _need_inputs(q, k, v, log_alpha, beta):
    """q, k [*lead, Dk] and v [*lead, Dv] in one dtype (bf16 or fp32), log_alpha [*lead, Dk] and
    beta [*lead] fp32, all contiguous on q's device."""
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dev, q.dtype)
    _dtype_code(q)
    _need(log_alpha, "log_alpha", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    lead, Dk = tuple(q.shape[:-1]), q.shape[-1]
    if tuple(k.shape) != lead + (Dk,) or tuple(log_alpha.shape) != lead + (Dk,) or \
            tuple(v.shape[:-1]) != lead or tuple(beta.shape) != lead:
        raise ValueError("inconsistent q/k/v/log_alpha/beta shapes")


def _out(t, name: str, device, dtype, shape):
    """A caller-provided output (or None -> a new tensor): the call writes `shape` elements of
    `dtype` through it."""
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _need(t, name, device, dtype)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _workspace(ws, device, nbytes: int):
    """The caller's workspace when it is a contiguous device buffer of at least `nbytes` bytes,
    else a new one. Returns (tensor, its size in bytes)."""
    if ws is not None:
        _need(ws, "workspace", device)
        if ws.numel() * ws.element_size() >= nbytes:
            return ws, ws.numel() * ws.element_size()
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    return ws, ws.numel()


def _size_dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"dtype {dtype} not supported (bf16 or fp32)")


def kda_chunk_fwd_workspace_size(B: int, T: int, H: int, Dk: int, Dv: int, chunk: int,
                                 num_seqs: int, dtype: torch.dtype) -> int:
    out = ctypes.c_size_t(0)
    code = _size_dtype_code(dtype)
    _check(lib().kda_chunk_fwd_workspace_size(B, T, H, Dk, Dv, chunk, num_seqs, code,
                                              ctypes.byref(out)), "kda_chunk_fwd_workspace_size")
    return int(out.value)


def _fusion(fusion, dev, H, Dk, o_like=None):
    """dict(qk_l2norm=bool, eps=float, A_log=[H] fp32, dt_bias=[H,Dk] fp32, out_norm=bool,
    out_norm_eps=float, out_norm_weight=[Dv] fp32, out_gate=o-shaped) -> kda_fusion_t."""
    if fusion is None:
        return None
    w, og = fusion.get("out_norm_weight"), fusion.get("out_gate")
    if fusion.get("out_norm"):
        if w is not None:
            _need(w, "out_norm_weight", dev, torch.float32)
            if o_like is not None and w.numel() != o_like.shape[-1]:
                raise ValueError("out_norm_weight must have Dv entries")
        if og is not None:
            _need(og, "out_gate", dev, o_like.dtype if o_like is not None else None)
            if o_like is not None and tuple(og.shape) != tuple(o_like.shape):
                raise ValueError("out_gate must have o's shape")
    else:
        w = og = None
    A_log, dt_bias = fusion.get("A_log"), fusion.get("dt_bias")
    if A_log is not None:
        _need(A_log, "A_log", dev, torch.float32)
        if A_log.numel() != H:
            raise ValueError("A_log must have H entries")
    if dt_bias is not None:
        _need(dt_bias, "dt_bias", dev, torch.float32)
        if dt_bias.numel() != H * Dk:
            raise ValueError("dt_bias must be [H, Dk]")
    return Fusion(1 if fusion.get("qk_l2norm") else 0, float(fusion.get("eps", 1e-6)),
                  None if A_log is None else A_log.data_ptr(),
                  None if dt_bias is None else dt_bias.data_ptr(),
                  1 if fusion.get("out_norm") else 0, float(fusion.get("out_norm_eps", 1e-5)),
                  None if w is None else w.data_ptr(), None if og is None else og.data_ptr())


def _prefill_checks(q, k, v, log_alpha, beta, initial_state, cu_seqlens) -> int:
    """Checks of the prefill inputs ([B,T,H,D] layout); returns the number of sequences N."""
    dev = q.device
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,Dk]")
    _need_inputs(q, k, v, log_alpha, beta)
    B, _, H, Dk = q.shape
    Dv = v.shape[-1]
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", dev, torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if initial_state is not None:
        _need(initial_state, "initial_state", dev, torch.float32)
        if tuple(initial_state.shape) != (N, H, Dk, Dv):
            raise ValueError("initial_state must be [N,H,Dk,Dv]")
    return N


def kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk: int = 64,
                  output_final_state: bool = True, o=None, final_state=None, workspace=None,
                  fusion=None):
    """Chunkwise KDA prefill.

    q, k [B,T,H,Dk], v [B,T,H,Dv] (bf16 or fp32, same dtype); log_alpha [B,T,H,Dk] fp32;
    beta [B,T,H] fp32; initial_state [N,H,Dk,Dv] fp32 or None; cu_seqlens int32 [N+1] on the
    device or None (then N = B). Returns (o [B,T,H,Dv] in the input dtype, final_state or None).
    ``fusion`` (dict, optional): qk_l2norm / eps normalise q and k in-kernel; A_log [H] and
    dt_bias [H,Dk] turn ``log_alpha`` (then the raw gate) into -exp(A_log) * softplus(g + dt_bias);
    out_norm / out_norm_eps / out_norm_weight [Dv] fp32 / out_gate (o's shape and dtype) make the
    stored output sigmoid(out_gate) * weight * o / sqrt(mean(o^2) + eps) per (token, head).
    """
    dev = q.device
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    N = _prefill_checks(q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    o = _out(o, "o", dev, q.dtype, (B, T, H, Dv))
    final_state = _out(final_state, "final_state", dev, torch.float32, (N, H, Dk, Dv)) \
        if output_final_state else None
    ws_bytes = kda_chunk_fwd_workspace_size(B, T, H, Dk, Dv, chunk, N, q.dtype)
    workspace, ws_len = _workspace(workspace, dev, ws_bytes)
    fz = _fusion(fusion, dev, H, Dk, v)
    args = (_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta),
            _ptr(initial_state), _ptr(cu_seqlens), N, B, T, H, Dk, Dv, chunk, _ptr(o),
            _ptr(final_state), _ptr(workspace), ws_len)
    with _on(dev):
        if fz is None:
            code = lib().kda_chunk_fwd(*args, _stream_handle(dev))
        else:
            code = lib().kda_chunk_fwd_fused(*args, ctypes.byref(fz), _stream_handle(dev))
    _check(code, "kda_chunk_fwd")
    return o, final_state


def kda_chunk_bwd_workspace_size(B: int, T: int, H: int, Dk: int, Dv: int, num_seqs: int,
                                 dtype: torch.dtype) -> int:
    out = ctypes.c_size_t(0)
    code = _size_dtype_code(dtype)
    _check(lib().kda_chunk_bwd_workspace_size(B, T, H, Dk, Dv, num_seqs, code, ctypes.byref(out)),
           "kda_chunk_bwd_workspace_size")
    return int(out.value)


def kda_chunk_bwd(q, k, v, log_alpha, beta, d_o, initial_state=None, d_final_state=None,
                  cu_seqlens=None, need_d_initial: bool = True, workspace=None):
    """Backward pass of :func:`kda_chunk_fwd` (same inputs, no fusion): gradients of
    <d_o, o> + <d_final_state, final_state>. Returns (dq, dk, dv in q's dtype, dlog_alpha and
    dbeta fp32, d_initial_state [N,H,Dk,Dv] fp32 or None)."""
    dev = q.device
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    N = _prefill_checks(q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    _need(d_o, "d_o", dev, q.dtype)
    if tuple(d_o.shape) != tuple(v.shape):
        raise ValueError("d_o must have v's shape")
    if d_final_state is not None:
        _need(d_final_state, "d_final_state", dev, torch.float32)
        if tuple(d_final_state.shape) != (N, H, Dk, Dv):
            raise ValueError("d_final_state must be [N,H,Dk,Dv]")
    dq, dk = torch.zeros_like(q), torch.zeros_like(k)
    dv = torch.zeros_like(v)
    dla = torch.zeros_like(log_alpha)
    db = torch.zeros_like(beta)
    ds0 = torch.empty((N, H, Dk, Dv), dtype=torch.float32, device=dev) if need_d_initial else None
    ws_bytes = kda_chunk_bwd_workspace_size(B, T, H, Dk, Dv, N, q.dtype)
    workspace, ws_len = _workspace(workspace, dev, ws_bytes)
    with _on(dev):
        code = lib().kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha),
                                   _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), N, B, T, H,
                                   Dk, Dv, _ptr(d_o), _ptr(d_final_state), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(dla), _ptr(db), _ptr(ds0), _ptr(workspace),
                                   ws_len, _stream_handle(dev))
    _check(code, "kda_chunk_bwd")
    return dq, dk, dv, dla, db, ds0


def kda_recurrent_step(q, k, v, log_alpha, beta, state, o=None, fusion=None):
    """One decode token per sequence: q, k [N,H,Dk], v [N,H,Dv], log_alpha [N,H,Dk] fp32,
    beta [N,H] fp32; ``state`` [N,H,Dk,Dv] fp32 is updated in place. Returns o [N,H,Dv].
    ``fusion``: as for :func:`kda_chunk_fwd` (out_gate then has o's shape [N,H,Dv])."""
    dev = q.device
    if q.dim() != 3:
        raise ValueError("q must be [N,H,Dk]")
    _need_inputs(q, k, v, log_alpha, beta)
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    _need(state, "state", dev, torch.float32)
    if tuple(state.shape) != (N, H, Dk, Dv):
        raise ValueError("state must be [N,H,Dk,Dv]")
    o = _out(o, "o", dev, q.dtype, (N, H, Dv))
    fz = _fusion(fusion, dev, H, Dk, v)
    args = (_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta), _ptr(state),
            _ptr(o), N, H, Dk, Dv)
    with _on(dev):
        if fz is None:
            code = lib().kda_recurrent_step(*args, _stream_handle(dev))
        else:
            code = lib().kda_recurrent_step_fused(*args, ctypes.byref(fz), _stream_handle(dev))
    _check(code, "kda_recurrent_step")
    return o


def kda_recurrent_fwd(q, k, v, log_alpha, beta, state_pool, state_indices=None, o=None,
                      fusion=None):
    """Token-by-token KDA over short sequences with states from a pool (serving-cache layout).

    q, k [N,T,H,Dk], v [N,T,H,Dv] (bf16 or fp32); log_alpha [N,T,H,Dk] fp32; beta [N,T,H] fp32;
    state_pool [P,H,Dk,Dv] fp32 updated in place; state_indices int32 [N] on the device (negative
    entries skip their sequence) or None for pool rows 0..N-1. Returns o [N,T,H,Dv]."""
    dev = q.device
    if q.dim() != 4:
        raise ValueError("q must be [N,T,H,Dk]")
    _need_inputs(q, k, v, log_alpha, beta)
    N, T, H, Dk = q.shape
    Dv = v.shape[-1]
    _need(state_pool, "state_pool", dev, torch.float32)
    P = state_pool.shape[0]
    if tuple(state_pool.shape[1:]) != (H, Dk, Dv):
        raise ValueError("state_pool must be [P,H,Dk,Dv]")
    if state_indices is not None:
        _need(state_indices, "state_indices", dev, torch.int32)
        if state_indices.numel() != N:
            raise ValueError("state_indices must have N entries")
    o = _out(o, "o", dev, q.dtype, (N, T, H, Dv))
    fz = _fusion(fusion, dev, H, Dk, v)
    args = (_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta),
            _ptr(state_pool), _ptr(state_indices), _ptr(o), N, T, H, Dk, Dv, P)
    with _on(dev):
        if fz is None:
            code = lib().kda_recurrent_fwd(*args, _stream_handle(dev))
        else:
            code = lib().kda_recurrent_fwd_fused(*args, ctypes.byref(fz), _stream_handle(dev))
    _check(code, "kda_recurrent_fwd")
    return o


def kda_last_device_error(device=None) -> int:
    """Read and clear the device status word (synchronises the current stream)."""
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    with _on(dev):
        return int(lib().kda_last_device_error(_stream_handle(dev)))


def kda_selftest_wait_timeout(limit_ns: int = 10_000_000, device=None) -> None:
    """Run the bounded-wait give-up path on purpose (include/kda_selftest.h): one block waits on
    an mbarrier phase that nothing completes and gives up after ``limit_ns``; the timeout is then
    reported by :func:`kda_last_device_error` on the same device."""
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    with _on(dev):
        code = lib().kda_selftest_wait_timeout(int(limit_ns), _stream_handle(dev))
    _check(code, "kda_selftest_wait_timeout")


def kda_profile_enable(enable: bool = True) -> None:
    """Bracket every kernel this library launches (from this thread) with CUDA events."""
    _check(lib().kda_profile_enable(1 if enable else 0), "kda_profile_enable")


def kda_profile_read() -> list[dict]:
    """Per-kernel launches and summed device ms since the last read (synchronises the events)."""
    cap = 64
    arr = (ProfileEntry * cap)()
    n = ctypes.c_int32(0)
    _check(lib().kda_profile_read(arr, cap, ctypes.byref(n)), "kda_profile_read")
    return [dict(name=arr[i].name.decode(), launches=int(arr[i].launches),
                 total_ms=float(arr[i].total_ms)) for i in range(min(n.value, cap))]


NOALLOC_SCRATCH_BYTES = 64 << 20  # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h


def kda_chunk_fwd_noalloc(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                          chunk: int = 64, o=None, final_state=None):
    """kda_chunk_fwd without a workspace, for callers that cannot allocate device scratch: the
    library uses its own fixed array of NOALLOC_SCRATCH_BYTES per GPU. Calls that need more are
    rejected (KDA_ERR_WORKSPACE); overlapping calls on one GPU race on the shared array. The
    outputs ``o`` / ``final_state`` may be passed in so that nothing is allocated here either."""
    dev = q.device
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    N = _prefill_checks(q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    o = _out(o, "o", dev, q.dtype, (B, T, H, Dv))
    final_state = _out(final_state, "final_state", dev, torch.float32, (N, H, Dk, Dv))
    with _on(dev):  # the scratch array used is the current device's
        code = lib().kda_chunk_fwd_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta),
            _ptr(initial_state), _ptr(cu_seqlens), N, B, T, H, Dk, Dv, chunk, _ptr(o),
            _ptr(final_state), _stream_handle(dev))
    _check(code, "kda_chunk_fwd_noalloc")
    return o, final_state
