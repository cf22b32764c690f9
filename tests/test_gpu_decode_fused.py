"""GPU parity of the fused decode step (kda_recurrent_step with the prologue and epilogue of
kda_fusion_t) against the fp64 oracle's prologue, one-token recurrence and output epilogue, on
the streaming kernel (bf16, d = 128) and on the token-by-token fallback (odd sizes)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import oracle
from tests._parity import TOL_DECODE_O, TOL_DECODE_S, rel_err, to_np
from tests.test_gpu_output_epilogue import epilogue_err

pytestmark = pytest.mark.gpu


def _step_inputs(N, H, Dk, Dv, seed, dev):
    g = torch.Generator(device=dev).manual_seed(seed)
    q = (torch.randn((N, H, Dk), generator=g, device=dev) * 3).to(torch.bfloat16)
    k = (torch.randn((N, H, Dk), generator=g, device=dev) * 3).to(torch.bfloat16)
    v = torch.randn((N, H, Dv), generator=g, device=dev).to(torch.bfloat16)
    gate = torch.randn((N, H, Dk), generator=g, device=dev) - 1.0
    beta = torch.sigmoid(torch.randn((N, H), generator=g, device=dev))
    og = (torch.randn((N, H, Dv), generator=g, device=dev) * 2).to(torch.bfloat16)
    return q, k, v, gate, beta, og


def _params(H, Dk, Dv, seed, dev):
    g = torch.Generator(device=dev).manual_seed(seed)
    A_log = torch.log(torch.rand((H,), generator=g, device=dev) * 15 + 1) - 2.0
    dt_bias = torch.randn((H, Dk), generator=g, device=dev) * 0.5
    w = torch.rand((Dv,), generator=g, device=dev) + 0.5
    return A_log, dt_bias, w


@pytest.mark.parametrize("dims", [(128, 128), (36, 20)])
@pytest.mark.parametrize("parts", ["prologue+epilogue", "prologue", "epilogue"])
def test_fused_decode_steps(cuda_device, dims, parts):
    """Five consecutive decode steps; dims (128, 128) run the streaming kernel, (36, 20) the
    token-by-token fallback (vectors not a multiple of 16 bytes)."""
    Dk, Dv = dims
    N, H, steps = 6, 3, 5
    A_log, dt_bias, w = _params(H, Dk, Dv, 1100, cuda_device)
    state = torch.randn((N, H, Dk, Dv), device=cuda_device) * 0.05
    S_ref = state.cpu().double().numpy()
    for t in range(steps):
        q, k, v, gate, beta, og = _step_inputs(N, H, Dk, Dv, 1110 + t, cuda_device)
        fz = {}
        if "prologue" in parts:
            fz.update(qk_l2norm=True, eps=1e-6, A_log=A_log, dt_bias=dt_bias)
        else:  # unit keys and a log decay as the plain operator expects
            q = (q.float() / q.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
            k = (k.float() / k.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
            gate = -torch.nn.functional.softplus(gate) * 0.5
        if "epilogue" in parts:
            fz.update(out_norm=True, out_norm_eps=1e-5, out_norm_weight=w, out_gate=og)
        y = kda.kda_recurrent_step(q, k, v, gate, beta, state, fusion=fz)
        torch.cuda.synchronize()
        assert kda.kda_last_device_error() == kda.KDA_OK
        qn, kn, la = oracle.prologue(q.cpu(), k.cpu(), gate.cpu(),
                                     A_log=A_log.cpu() if "prologue" in parts else None,
                                     dt_bias=dt_bias.cpu() if "prologue" in parts else None,
                                     qk_l2norm="prologue" in parts, eps=1e-6)
        o_ref, S_ref = oracle.recurrent(qn, kn, v.cpu(), la, beta.cpu(), initial_state=S_ref,
                                        cu_seqlens=np.arange(N + 1))
        if "epilogue" in parts:
            y_ref = oracle.output_norm_gate(o_ref, to_np(og), to_np(w), 1e-5)
            assert epilogue_err(y, y_ref, o_ref, fz, H) <= TOL_DECODE_O, t
        else:
            assert rel_err(y, o_ref) <= TOL_DECODE_O, t
        assert rel_err(state, S_ref) <= TOL_DECODE_S, t


def test_fused_decode_without_options_equals_plain_step(cuda_device):
    N, H = 4, 2
    q, k, v, gate, beta, _ = _step_inputs(N, H, 128, 128, 1120, cuda_device)
    q = (q.float() / q.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    k = (k.float() / k.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    la = -torch.nn.functional.softplus(gate) * 0.5
    s0 = torch.randn((N, H, 128, 128), device=cuda_device) * 0.05
    sa, sb = s0.clone(), s0.clone()
    a = kda.kda_recurrent_step(q, k, v, la, beta, sa)
    b = kda.kda_recurrent_step(q, k, v, la, beta, sb, fusion={})
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(sa, sb)
