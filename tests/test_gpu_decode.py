"""GPU parity of kda_recurrent_step (decode) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
import oracle
from tests._parity import TOL_DECODE_O, TOL_DECODE_S, TOL_F32, rel_err, to_np

pytestmark = pytest.mark.gpu


def _oracle_steps(state0, steps: dict, n_steps: int, seq_idx=None):
    """Run the oracle token by token: each decode step is a one-token sequence per (n, h)."""
    S = to_np(state0)
    if seq_idx is not None:
        S = S[seq_idx]
    outs = []
    for s in range(n_steps):
        sel = (lambda t: t[s] if seq_idx is None else t[s][seq_idx])
        q, k, v, la, b = (sel(steps[x]) for x in ("q", "k", "v", "log_alpha", "beta"))
        N = q.shape[0]
        cu = np.arange(N + 1, dtype=np.int64)
        o, S = oracle.recurrent(q, k, v, la, b, initial_state=S, cu_seqlens=cu)
        outs.append(o)
    return np.stack(outs), S


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dims", [(128, 128), (40, 12), (128, 64), (1, 4)])
def test_decode_small(cuda_device, dtype, dims):
    Dk, Dv = dims
    spec = kda_synth.DecodeSpec("t", N=5, H=3, Dk=Dk, Dv=Dv, steps=6, dtype=dtype, decay="fast",
                                init_std=0.02)
    state = kda_synth.decode_state(spec, 7, cuda_device)
    steps = kda_synth.decode_step_inputs(spec, 7, spec.steps, cuda_device)
    state0 = state.clone()
    outs = []
    for s in range(spec.steps):
        outs.append(kda.kda_recurrent_step(steps["q"][s], steps["k"][s], steps["v"][s],
                                           steps["log_alpha"][s], steps["beta"][s], state))
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle_steps(state0, steps, spec.steps)
    tol_o = TOL_DECODE_O if dtype == "bf16" else TOL_F32
    assert rel_err(torch.stack(outs), o_ref) <= tol_o
    assert rel_err(state, S_ref) <= TOL_DECODE_S


def test_decode_full_size_sampled(cuda_device):
    """The decode workload's full size (256 sequences x 32 heads, 128 x 128 fp32 states) for a
    run of steps; o at every step and the final states of 16 sampled sequences (all heads) are
    compared with the oracle, and every state stays finite."""
    spec = kda_synth.DECODE
    n_steps = 64
    state = kda_synth.decode_state(spec, 2004, cuda_device)
    steps = kda_synth.decode_step_inputs(spec, 2004, n_steps, cuda_device)
    pick = np.sort(np.random.default_rng(0).choice(spec.N, 16, replace=False))
    state0 = state[pick].cpu()
    outs = []
    for s in range(n_steps):
        o = kda.kda_recurrent_step(steps["q"][s], steps["k"][s], steps["v"][s],
                                   steps["log_alpha"][s], steps["beta"][s], state)
        outs.append(o[pick].cpu())
    torch.cuda.synchronize()
    host = {k: v[:, pick].cpu() for k, v in steps.items()}
    o_ref, S_ref = _oracle_steps(state0, host, n_steps)
    assert rel_err(torch.stack(outs), o_ref) <= TOL_DECODE_O
    assert rel_err(state[pick], S_ref) <= TOL_DECODE_S
    assert torch.isfinite(state).all()


def test_decode_all_steps_sampled(cuda_device):
    """The decode workload end to end: 256 sequences x 32 heads, all of its 1024 steps on the
    same in-place states. Inputs are drawn 64 steps at a time (step s from its own seed, as in
    one 1024-step draw); 16 sampled sequences (all heads) follow in the oracle, o compared at
    every step and the states after the last one."""
    spec = kda_synth.DECODE
    block = 64
    state = kda_synth.decode_state(spec, 2005, cuda_device)
    pick = np.sort(np.random.default_rng(1).choice(spec.N, 16, replace=False))
    S_ref = to_np(state[pick])
    worst_o = 0.0
    for b in range(spec.steps // block):
        steps = kda_synth.decode_step_inputs(spec, 2005 + block * b, block, cuda_device)
        outs = []
        for s in range(block):
            o = kda.kda_recurrent_step(steps["q"][s], steps["k"][s], steps["v"][s],
                                       steps["log_alpha"][s], steps["beta"][s], state)
            outs.append(o[pick].cpu())
        torch.cuda.synchronize()
        host = {k: v[:, pick].cpu() for k, v in steps.items()}
        o_ref, S_ref = _oracle_steps(S_ref, host, block)
        worst_o = max(worst_o, rel_err(torch.stack(outs), o_ref))
        del steps
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert worst_o <= TOL_DECODE_O, worst_o
    assert rel_err(state[pick], S_ref) <= TOL_DECODE_S
    assert torch.isfinite(state).all()


def test_decode_is_deterministic(cuda_device):
    spec = kda_synth.DecodeSpec("t", N=64, H=8, Dk=128, Dv=128, steps=1, dtype="bf16",
                                decay="slow", init_std=0.02)
    s1 = kda_synth.decode_state(spec, 3, cuda_device)
    s2 = s1.clone()
    st = kda_synth.decode_step_inputs(spec, 3, 1, cuda_device)
    a = kda.kda_recurrent_step(st["q"][0], st["k"][0], st["v"][0], st["log_alpha"][0],
                               st["beta"][0], s1)
    b = kda.kda_recurrent_step(st["q"][0], st["k"][0], st["v"][0], st["log_alpha"][0],
                               st["beta"][0], s2)
    assert torch.equal(a, b) and torch.equal(s1, s2)
