"""Shared helpers of the GPU parity tests: tolerances and error metrics.

Tolerances (max-abs error relative to the largest oracle magnitude over the compared tensor):
  fp32 inputs (CUDA-core path): o and final state within 1e-4.
  bf16 inputs, fp32 state and accumulation (tensor-core path): o within 2e-2; final state within
  2e-2 (bf16 operands feed the correction terms of the state update).
  decode (fp32 arithmetic on bf16-rounded inputs): o within 2e-2 in bf16 output, state within 1e-4.
"""
import numpy as np
import torch

TOL_F32 = 1e-4
TOL_BF16_O = 2e-2
TOL_BF16_S = 2e-2
TOL_DECODE_O = 2e-2
TOL_DECODE_S = 1e-4


def to_np(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.double().numpy()


def rel_err(got, ref) -> float:
    got, ref = to_np(got), to_np(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = float(np.abs(ref).max())
    if scale == 0.0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max()) / scale


def cu_list(B, T):
    return np.arange(B + 1, dtype=np.int64) * T
