"""fp64 CPU oracle of the Kimi Delta Attention operator — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
package. The CUDA library never calls it, links it or shares code with it.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64, OpenMP over sequence x head); this
module compiles it with gcc on first use and marshals numpy / torch arrays into fp64 buffers.

Functions
  recurrent(...)           the token-by-token definition: Eq. 1 of "Kimi Linear: An Expressive,
                           Efficient Attention Architecture" (paper-graph-ui walkthrough, §3.4
                           "The KDA State Update Equation") with the read o_t = S_t^T q_t.
  chunked(...)             the chunkwise WY/UT evaluation of §3.4 "Chunkwise Parallelization"
                           (Eq. 8, Eq. 9), fp64; pins the chunk algebra against ``recurrent``.
  unit_lower_inverse(A)    (I + A)^{-1} by forward substitution (the UT transform's inverse).
  recurrent_bwd(...)       reverse-mode derivative of ``recurrent`` (the backward pass): gradients
                           of <d_o, o> + <d_final, S_T> with respect to every input.
  prologue(...)            the fused input steps: L2-normalised q, k and the log-space decay gate
                           log alpha = -exp(A_log[h]) * softplus(g + dt_bias[h, c]) (walkthrough
                           §3.4 "Neural Parameterization"; the L2 Deep Distill page's
                           implementation notes on the in-kernel L2 norm and the fused gate).
  output_norm_gate(...)    the output epilogue y = sigmoid(gate) * weight * o / RMS(o), the RMS
                           taken over the value channels of each (token, head) (walkthrough §3.4
                           "Neural Parameterization", the output-gate equation; the L2 Deep
                           Distill page's module table: FusedRMSNormGated, sigmoid gate inside the
                           RMSNorm).

All inputs follow the packed layout [T_total, H, D] with int64 ``cu_seqlens`` [N+1]; a batch of B
equal-length sequences is the same memory as [B, T, H, D] with cu_seqlens = [0, T, 2T, ...].
Every function here has parity pins in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into libkda_oracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            sig = [_dp, _dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_int64, ctypes.c_int64]
            lib.kda_oracle_recurrent.argtypes = sig + [_dp, _dp, ctypes.c_int]
            lib.kda_oracle_recurrent.restype = ctypes.c_int
            lib.kda_oracle_chunked.argtypes = sig + [ctypes.c_int64, _dp, _dp, ctypes.c_int]
            lib.kda_oracle_chunked.restype = ctypes.c_int
            lib.kda_oracle_unit_lower_inverse.argtypes = [_dp, ctypes.c_int64, _dp]
            lib.kda_oracle_unit_lower_inverse.restype = None
            lib.kda_oracle_recurrent_bwd.argtypes = sig + [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                                            ctypes.c_int]
            lib.kda_oracle_recurrent_bwd.restype = ctypes.c_int
            lib.kda_oracle_max_threads.argtypes = []
            lib.kda_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    """OpenMP threads the oracle uses by default on this host."""
    return int(_load().kda_oracle_max_threads())


def _f64(x) -> np.ndarray:
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> contiguous fp64 numpy."""
    if hasattr(x, "detach"):  # torch tensor; bf16 has no numpy dtype, widen through fp32
        import torch

        t = x.detach().to("cpu")
        if t.dtype in (torch.bfloat16, torch.float16):
            t = t.float()
        x = t.double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def _prep(q, k, v, log_alpha, beta, initial_state, cu_seqlens):
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    H, Dk = q.shape[-2], q.shape[-1]
    Dv = v.shape[-1]
    q = q.reshape(-1, H, Dk)
    k = k.reshape(-1, H, Dk)
    la = la.reshape(-1, H, Dk)
    v = v.reshape(-1, H, Dv)
    b = b.reshape(-1, H)
    T = q.shape[0]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    s0 = None if initial_state is None else _f64(initial_state).reshape(N, H, Dk, Dv)
    for a, shp in ((k, (T, H, Dk)), (la, (T, H, Dk)), (v, (T, H, Dv)), (b, (T, H))):
        if a.shape != shp:
            raise ValueError(f"oracle: shape {a.shape} != {shp}")
    if cu[0] != 0 or np.any(np.diff(cu) < 0) or cu[-1] > T:
        raise ValueError("oracle: bad cu_seqlens")
    return q, k, v, la, b, s0, cu, N, H, Dk, Dv


def recurrent(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, nthreads: int = 0):
    """Token-by-token fp64 recurrence. Returns (o [T_total,H,Dv], final_state [N,H,Dk,Dv]).

    Inputs may be [T_total, H, D] or [B, T, H, D]; with ``cu_seqlens=None`` they form ONE
    sequence of T_total tokens (pass cu_seqlens=[0,T,2T,...] for a batch of B sequences).
    """
    q, k, v, la, b, s0, cu, N, H, Dk, Dv = _prep(q, k, v, log_alpha, beta, initial_state,
                                                 cu_seqlens)
    o = np.zeros((q.shape[0], H, Dv), dtype=np.float64)
    s = np.zeros((N, H, Dk, Dv), dtype=np.float64)
    rc = _load().kda_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
                                      cu.ctypes.data_as(_i64p), N, H, Dk, Dv, _ptr(o), _ptr(s),
                                      int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle: kda_oracle_recurrent failed")
    return o, s


def chunked(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk: int = 64,
            nthreads: int = 0):
    """Chunkwise WY/UT evaluation (fp64), same contract as :func:`recurrent`."""
    q, k, v, la, b, s0, cu, N, H, Dk, Dv = _prep(q, k, v, log_alpha, beta, initial_state,
                                                 cu_seqlens)
    o = np.zeros((q.shape[0], H, Dv), dtype=np.float64)
    s = np.zeros((N, H, Dk, Dv), dtype=np.float64)
    rc = _load().kda_oracle_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
                                    cu.ctypes.data_as(_i64p), N, H, Dk, Dv, int(chunk), _ptr(o),
                                    _ptr(s), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle: kda_oracle_chunked failed")
    return o, s


def unit_lower_inverse(A) -> np.ndarray:
    """(I + StrictTril(A))^{-1} by forward substitution; A is C x C (its upper part is ignored)."""
    A = _f64(A)
    C = A.shape[0]
    A = np.ascontiguousarray(np.tril(A, -1))
    X = np.zeros((C, C), dtype=np.float64)
    _load().kda_oracle_unit_lower_inverse(_ptr(A), C, _ptr(X))
    return X


def _softplus(x: np.ndarray) -> np.ndarray:
    """log(1 + exp(x)), evaluated without overflow for large x."""
    return np.where(x > 30.0, x, np.log1p(np.exp(np.minimum(x, 30.0))))


def prologue(q, k, log_alpha_or_gate, A_log=None, dt_bias=None, qk_l2norm=False, eps=1e-6):
    """fp64 (q', k', log_alpha') after the optional in-kernel steps: q, k divided by
    sqrt(sum x^2 + eps) over the key channels of each (token, head); and, when A_log is given,
    log_alpha' = -exp(A_log[h]) * softplus(g + dt_bias[h, c]) with g = log_alpha_or_gate.
    Arrays keep their shapes (..., H, Dk)."""
    q, k, g = _f64(q), _f64(k), _f64(log_alpha_or_gate)
    if qk_l2norm:
        q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + eps)
        k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + eps)
    if A_log is not None:
        a = np.exp(_f64(A_log))  # [H]
        b = np.zeros(g.shape[-2:]) if dt_bias is None else _f64(dt_bias).reshape(g.shape[-2:])
        g = -a[:, None] * _softplus(g + b)
    return q, k, g


def _sigmoid(x: np.ndarray) -> np.ndarray:
    """1 / (1 + exp(-x)), evaluated without overflow for either sign."""
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def output_norm_gate(o, gate=None, weight=None, eps=1e-6):
    """fp64 y = sigmoid(gate) * weight * o / sqrt(mean_c(o_c^2) + eps) over the last axis (the
    value channels of one (token, head)); gate None means no gate, weight None means ones.
    ``o`` and ``gate`` share a shape (..., Dv); ``weight`` is [Dv]."""
    o = _f64(o)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    y = o / rms
    if weight is not None:
        y = y * _f64(weight).reshape(-1)
    if gate is not None:
        y = y * _sigmoid(_f64(gate).reshape(o.shape))
    return y


def recurrent_bwd(q, k, v, log_alpha, beta, d_o, initial_state=None, d_final=None,
                  cu_seqlens=None, nthreads: int = 0):
    """fp64 gradients (d_q, d_k, d_v, d_log_alpha, d_beta, d_initial) of
    L = <d_o, o> + <d_final, final_state> for the recurrence of :func:`recurrent` (same input
    conventions; d_o has o's shape, d_final the state's)."""
    q, k, v, la, b, s0, cu, N, H, Dk, Dv = _prep(q, k, v, log_alpha, beta, initial_state,
                                                 cu_seqlens)
    T = q.shape[0]
    do = _f64(d_o).reshape(T, H, Dv)
    dfin = None if d_final is None else _f64(d_final).reshape(N, H, Dk, Dv)
    dq = np.zeros((T, H, Dk)); dk = np.zeros((T, H, Dk)); dla = np.zeros((T, H, Dk))
    dv = np.zeros((T, H, Dv)); db = np.zeros((T, H)); ds0 = np.zeros((N, H, Dk, Dv))
    rc = _load().kda_oracle_recurrent_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
                                          cu.ctypes.data_as(_i64p), N, H, Dk, Dv, _ptr(do),
                                          _ptr(dfin), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla),
                                          _ptr(db), _ptr(ds0), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle: kda_oracle_recurrent_bwd failed")
    return dq, dk, dv, dla, db, ds0
