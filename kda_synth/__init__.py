"""Seeded synthetic inputs for the KDA operator (shared by the tests, the smoke check and bench.py).

This module holds only input distributions, never any of the operator's arithmetic. The same
tensors feed both the CUDA library and the fp64 oracle (copied to the host for the latter).

Distributions (per token and head unless stated):
  q, k       N(0,1) draws, L2-normalised per (token, head) vector in fp32, then rounded to the
             input dtype (bf16 round-to-nearest-even). The oracle consumes the ROUNDED values.
  v          N(0,1), rounded to the input dtype.
  log_alpha  per key channel, fp32:  "fast" decay  = -softplus(N(0,1)) * 0.5
                                     "slow" decay  = -softplus(N(-2,1))
  beta       sigmoid(N(0,1)), fp32.
  state      N(0, std^2) per element (std = 0.02 where the workload asks for it), else zeros.
  lengths    for packed variable-length batches: floor(exp(U(ln lo, ln hi))) clamped to [lo, hi],
             drawn with numpy's PCG64 from the same seed, packed in draw order.

Tensors are drawn with ``torch.Generator(device).manual_seed(seed)`` in a fixed order, so a
(spec, seed, device) triple always yields the same values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    """Shape and distribution of one chunkwise-prefill workload."""

    name: str
    B: int
    T: int  # tokens per sequence (or total tokens when seqlens is given)
    H: int
    Dk: int
    Dv: int
    chunk: int
    dtype: str  # "bf16" or "f32"
    decay: str  # "fast" or "slow"
    init_std: float  # 0.0 => zero initial state
    seqlens: Optional[Sequence[int]] = None  # packed varlen lengths (B must be 1)

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens) if self.seqlens is not None else self.B

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens)) if self.seqlens is not None else self.B * self.T

    def token_heads(self) -> int:
        return self.total_tokens * self.H


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    """Shape and distribution of the single-token recurrent decode workload."""

    name: str
    N: int
    H: int
    Dk: int
    Dv: int
    steps: int
    dtype: str
    decay: str
    init_std: float


def loguniform_lengths(n: int, lo: int, hi: int, seed: int) -> list[int]:
    """n lengths floor(exp(U(ln lo, ln hi))) clamped to [lo, hi] (numpy PCG64, seeded)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return [int(min(max(math.floor(math.exp(x)), lo), hi)) for x in u]


# The five workloads of the operator's evaluation (tiny fp32 parity case, standard prefill,
# long prefill, packed variable-length prefill, batched decode).
TINY = PrefillSpec("tiny_f32_T256_d32", B=1, T=256, H=1, Dk=32, Dv=32, chunk=64, dtype="f32",
                   decay="fast", init_std=0.0)
STANDARD = PrefillSpec("prefill_B2_T4096_H32_d128", B=2, T=4096, H=32, Dk=128, Dv=128, chunk=64,
                       dtype="bf16", decay="fast", init_std=0.02)
LONG = PrefillSpec("prefill_B1_T131072_H32_d128", B=1, T=131072, H=32, Dk=128, Dv=128, chunk=64,
                   dtype="bf16", decay="slow", init_std=0.0)


def varlen_spec(seed: int = 1003, n: int = 16, lo: int = 256, hi: int = 32768) -> PrefillSpec:
    lens = loguniform_lengths(n, lo, hi, seed)
    return PrefillSpec(f"varlen_{n}seq_H32_d128", B=1, T=int(sum(lens)), H=32, Dk=128, Dv=128,
                       chunk=64, dtype="bf16", decay="fast", init_std=0.0, seqlens=tuple(lens))


DECODE = DecodeSpec("decode_N256_H32_d128", N=256, H=32, Dk=128, Dv=128, steps=1024,
                    dtype="bf16", decay="slow", init_std=0.02)


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _log_alpha(shape, decay: str, g: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if decay == "fast":
        return -torch.nn.functional.softplus(z) * 0.5
    if decay == "slow":
        return -torch.nn.functional.softplus(z - 2.0)
    raise ValueError(decay)


def prefill_inputs(spec: PrefillSpec, seed: int, device="cpu") -> dict:
    """Draw one prefill batch. Returns a dict of tensors on ``device`` in the library layout:
    q, k [B,T,H,Dk], v [B,T,H,Dv] (spec dtype); log_alpha [B,T,H,Dk] f32; beta [B,T,H] f32;
    initial_state [N,H,Dk,Dv] f32 or None; cu_seqlens int32 [N+1] or None."""
    device = torch.device(device)
    g = _gen(device, seed)
    dt = torch_dtype(spec.dtype)
    B, T, H, Dk, Dv = spec.B, spec.T, spec.H, spec.Dk, spec.Dv
    q = _unit_rows(torch.randn((B, T, H, Dk), generator=g, device=device)).to(dt)
    k = _unit_rows(torch.randn((B, T, H, Dk), generator=g, device=device)).to(dt)
    v = torch.randn((B, T, H, Dv), generator=g, device=device).to(dt)
    log_alpha = _log_alpha((B, T, H, Dk), spec.decay, g, device)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, device=device))
    N = spec.num_seqs
    init = None
    if spec.init_std > 0:
        init = torch.randn((N, H, Dk, Dv), generator=g, device=device) * spec.init_std
    cu = None
    if spec.seqlens is not None:
        if B != 1:
            raise ValueError("packed varlen needs B == 1")
        offs = np.concatenate([[0], np.cumsum(np.asarray(spec.seqlens, dtype=np.int64))])
        cu = torch.tensor(offs, dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, initial_state=init, cu_seqlens=cu)


def decode_state(spec: DecodeSpec, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    return torch.randn((spec.N, spec.H, spec.Dk, spec.Dv), generator=g, device=device) * \
        spec.init_std


def decode_step_inputs(spec: DecodeSpec, seed: int, steps: int, device="cpu") -> dict:
    """Per-step decode inputs stacked along a leading step axis:
    q, k [steps,N,H,Dk], v [steps,N,H,Dv] (spec dtype); log_alpha [steps,N,H,Dk] f32;
    beta [steps,N,H] f32. Step s is drawn from seed + 1 + s so any prefix is reproducible."""
    device = torch.device(device)
    dt = torch_dtype(spec.dtype)
    N, H, Dk, Dv = spec.N, spec.H, spec.Dk, spec.Dv
    out = dict(q=torch.empty((steps, N, H, Dk), dtype=dt, device=device),
               k=torch.empty((steps, N, H, Dk), dtype=dt, device=device),
               v=torch.empty((steps, N, H, Dv), dtype=dt, device=device),
               log_alpha=torch.empty((steps, N, H, Dk), dtype=torch.float32, device=device),
               beta=torch.empty((steps, N, H), dtype=torch.float32, device=device))
    for s in range(steps):
        g = _gen(device, seed + 1 + s)
        out["q"][s] = _unit_rows(torch.randn((N, H, Dk), generator=g, device=device)).to(dt)
        out["k"][s] = _unit_rows(torch.randn((N, H, Dk), generator=g, device=device)).to(dt)
        out["v"][s] = torch.randn((N, H, Dv), generator=g, device=device).to(dt)
        out["log_alpha"][s] = _log_alpha((N, H, Dk), spec.decay, g, device)
        out["beta"][s] = torch.sigmoid(torch.randn((N, H), generator=g, device=device))
    return out
