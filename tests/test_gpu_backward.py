"""GPU parity of kda_chunk_bwd (the backward pass) against the fp64 oracle's reverse-mode
derivative of the recurrence (itself pinned by finite differences), through the C ABI."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
import oracle
from kda_synth import PrefillSpec
from tests._parity import TOL_F32, rel_err

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_initial")


def _cotangents(spec, N, seed, dev):
    g = torch.Generator(device=dev).manual_seed(seed)
    dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    d_o = torch.randn((spec.B, spec.T, spec.H, spec.Dv), generator=g, device=dev).to(dt)
    d_fin = torch.randn((N, spec.H, spec.Dk, spec.Dv), generator=g, device=dev)
    return d_o, d_fin


def _compare(inp, d_o, d_fin, cu, tol_qkv, tol_rest, H):
    got = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o,
                            initial_state=inp["initial_state"], d_final_state=d_fin,
                            cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    ref = oracle.recurrent_bwd(*(inp[x].cpu() for x in ("q", "k", "v", "log_alpha", "beta")),
                               d_o.cpu(), initial_state=None if inp["initial_state"] is None
                               else inp["initial_state"].cpu(), d_final=d_fin.cpu(),
                               cu_seqlens=cu)
    errs = {}
    for name, a, b in zip(NAMES, got, ref):
        a = a.reshape(b.shape) if name != "d_initial" else a
        errs[name] = rel_err(a, b)
        tol = tol_qkv if name in ("dq", "dk", "dv") else tol_rest
        assert errs[name] <= tol, f"{name}: {errs[name]:.3e} > {tol}"
    return errs


@pytest.mark.parametrize("T", [1, 31, 100])
def test_backward_f32_ragged(cuda_device, T):
    spec = PrefillSpec("t", B=2, T=T, H=2, Dk=48, Dv=20, chunk=64, dtype="f32", decay="fast",
                       init_std=0.5)
    inp = kda_synth.prefill_inputs(spec, 900 + T, cuda_device)
    d_o, d_fin = _cotangents(spec, 2, 901, cuda_device)
    _compare(inp, d_o, d_fin, np.arange(3) * T, TOL_F32, TOL_F32, 2)


def test_backward_f32_varlen_with_empty_sequences(cuda_device):
    lens = [5, 70, 0, 33]
    T = sum(lens)
    spec = PrefillSpec("t", B=1, T=T, H=2, Dk=32, Dv=32, chunk=64, dtype="f32", decay="fast",
                       init_std=0.5, seqlens=tuple(lens))
    inp = kda_synth.prefill_inputs(spec, 910, cuda_device)
    inp["initial_state"] = torch.randn((len(lens), 2, 32, 32), device=cuda_device) * 0.5
    d_o, d_fin = _cotangents(spec, len(lens), 911, cuda_device)
    errs = _compare(inp, d_o, d_fin, inp["cu_seqlens"].cpu().numpy(), TOL_F32, TOL_F32, 2)
    assert all(np.isfinite(list(errs.values())))


def test_backward_f32_strong_decay(cuda_device):
    """Per-token decays down to exp(-20): every ratio in the backward stays exp(g_r - g_i) <= 1."""
    spec = PrefillSpec("t", B=1, T=96, H=2, Dk=32, Dv=16, chunk=64, dtype="f32", decay="fast",
                       init_std=0.5)
    inp = kda_synth.prefill_inputs(spec, 920, cuda_device)
    inp["log_alpha"] = inp["log_alpha"] * 40.0
    d_o, d_fin = _cotangents(spec, 1, 921, cuda_device)
    _compare(inp, d_o, d_fin, np.array([0, 96]), TOL_F32, TOL_F32, 2)


@pytest.mark.parametrize("T", [300, 4096])
def test_backward_bf16_d128(cuda_device, T):
    """bf16 inputs, fp32 arithmetic: dq, dk, dv come back in bf16 (2e-2); the fp32 gradients are
    held to 1e-3. T = 4096 runs 128 backward chunks through the state pass."""
    spec = PrefillSpec("t", B=1, T=T, H=2 if T > 1000 else 3, Dk=128, Dv=128, chunk=64,
                       dtype="bf16", decay="fast", init_std=0.02)
    inp = kda_synth.prefill_inputs(spec, 930 + T, cuda_device)
    d_o, d_fin = _cotangents(spec, 1, 931, cuda_device)
    _compare(inp, d_o, d_fin, np.array([0, T]), 2e-2, 1e-3, spec.H)


def test_backward_without_final_cotangent_or_initial_state(cuda_device):
    spec = PrefillSpec("t", B=2, T=40, H=1, Dk=16, Dv=16, chunk=64, dtype="f32", decay="slow",
                       init_std=0.0)
    inp = kda_synth.prefill_inputs(spec, 940, cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(941)
    d_o = torch.randn((2, 40, 1, 16), generator=g, device=cuda_device)
    got = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o)
    torch.cuda.synchronize()
    ref = oracle.recurrent_bwd(*(inp[x].cpu() for x in ("q", "k", "v", "log_alpha", "beta")),
                               d_o.cpu(), cu_seqlens=np.array([0, 40, 80]))
    for name, a, b in zip(NAMES, got, ref):
        assert rel_err(a.reshape(b.shape), b) <= TOL_F32, name


def test_backward_is_deterministic(cuda_device):
    spec = PrefillSpec("t", B=1, T=200, H=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                       decay="fast", init_std=0.02)
    inp = kda_synth.prefill_inputs(spec, 950, cuda_device)
    d_o, d_fin = _cotangents(spec, 1, 951, cuda_device)
    a = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o,
                          initial_state=inp["initial_state"], d_final_state=d_fin)
    b = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o,
                          initial_state=inp["initial_state"], d_final_state=d_fin)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
