"""GPU parity of the fused prologue (in-kernel q/k L2 normalisation and the log-space decay gate)
on the chunkwise and recurrent paths, against the fp64 oracle's prologue + recurrence."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import oracle
from tests._parity import TOL_BF16_O, TOL_BF16_S, TOL_DECODE_O, TOL_DECODE_S, TOL_F32, rel_err

pytestmark = pytest.mark.gpu


def _raw_inputs(B, T, H, Dk, Dv, dtype, seed, dev):
    """Un-normalised q, k (scale ~3) and raw gates, as the projections would produce them."""
    g = torch.Generator(device=dev).manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = (torch.randn((B, T, H, Dk), generator=g, device=dev) * 3.0).to(dt)
    k = (torch.randn((B, T, H, Dk), generator=g, device=dev) * 3.0).to(dt)
    v = torch.randn((B, T, H, Dv), generator=g, device=dev).to(dt)
    gate = torch.randn((B, T, H, Dk), generator=g, device=dev) - 1.0
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, device=dev))
    A_log = torch.log(torch.rand((H,), generator=g, device=dev) * 15.0 + 1.0) - 2.0
    dt_bias = torch.randn((H, Dk), generator=g, device=dev) * 0.5
    return dict(q=q, k=k, v=v, gate=gate, beta=beta, A_log=A_log, dt_bias=dt_bias)


def _oracle_fused(x, fusion, initial_state, cu):
    q, k, la = oracle.prologue(x["q"].cpu(), x["k"].cpu(), x["gate"].cpu(),
                               A_log=x["A_log"].cpu() if fusion.get("A_log") is not None else None,
                               dt_bias=x["dt_bias"].cpu()
                               if fusion.get("dt_bias") is not None else None,
                               qk_l2norm=bool(fusion.get("qk_l2norm")), eps=fusion.get("eps", 1e-6))
    H = q.shape[-2]
    return oracle.recurrent(q.reshape(-1, H, q.shape[-1]), k.reshape(-1, H, k.shape[-1]),
                            x["v"].cpu(), la.reshape(-1, H, la.shape[-1]), x["beta"].cpu(),
                            initial_state=initial_state, cu_seqlens=cu)


@pytest.mark.parametrize("mode", ["l2+gate", "l2", "gate"])
def test_chunk_fused_bf16(cuda_device, mode):
    B, T, H = 2, 200, 3
    x = _raw_inputs(B, T, H, 128, 128, "bf16", 700, cuda_device)
    fusion = {"eps": 1e-6}
    if "l2" in mode:
        fusion["qk_l2norm"] = True
    if "gate" in mode:
        fusion.update(A_log=x["A_log"], dt_bias=x["dt_bias"])
    else:  # without the fused gate the decay input must already be a log decay
        x["gate"] = -torch.nn.functional.softplus(x["gate"]) * 0.5
    if mode == "gate":  # without the fused norm, feed unit-norm keys as the operator expects
        x["q"] = (x["q"].float() / x["q"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        x["k"] = (x["k"].float() / x["k"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    s0 = torch.randn((B, H, 128, 128), device=cuda_device) * 0.02
    o, s = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["gate"], x["beta"], initial_state=s0,
                             chunk=64, fusion=fusion)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    o_ref, s_ref = _oracle_fused(x, fusion, s0.cpu(), np.arange(B + 1) * T)
    assert rel_err(o.reshape(-1, H, 128), o_ref) <= TOL_BF16_O
    assert rel_err(s, s_ref) <= TOL_BF16_S


def test_chunk_decays_between_the_two_bounds(cuda_device):
    """Chunks whose strongest channels decay by exp(-70) over 64 tokens: with the in-kernel L2
    norm (|k| <= 1) they take the single-reference evaluation (bound exp(-80)), with caller-
    normalised keys the block-reference one (bound exp(-60)); both match the oracle."""
    B, T, H = 1, 250, 2
    x = _raw_inputs(B, T, H, 128, 128, "bf16", 710, cuda_device)
    la = -torch.nn.functional.softplus(x["gate"]) * 0.5
    la[..., :16] = -70.0 / 64.0
    x["gate"] = la
    s0 = torch.randn((B, H, 128, 128), device=cuda_device) * 0.02
    qn = (x["q"].float() / x["q"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    kn = (x["k"].float() / x["k"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    for fusion, q, k in (({"eps": 1e-6, "qk_l2norm": True}, x["q"], x["k"]), ({}, qn, kn)):
        o, s = kda.kda_chunk_fwd(q, k, x["v"], la, x["beta"], initial_state=s0, chunk=64,
                                 fusion=fusion or None)
        torch.cuda.synchronize()
        assert kda.kda_last_device_error() == kda.KDA_OK
        y = dict(x, q=q, k=k)
        o_ref, s_ref = _oracle_fused(y, fusion, s0.cpu(), np.array([0, T]))
        assert rel_err(o.reshape(-1, H, 128), o_ref) <= TOL_BF16_O
        assert rel_err(s, s_ref) <= TOL_BF16_S


def test_chunk_fused_f32_varlen(cuda_device):
    lens = [5, 70, 0, 33]
    T, H, Dk, Dv = sum(lens), 2, 48, 20
    x = _raw_inputs(1, T, H, Dk, Dv, "f32", 710, cuda_device)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32,
                      device=cuda_device)
    fusion = dict(qk_l2norm=True, eps=1e-6, A_log=x["A_log"], dt_bias=x["dt_bias"])
    o, s = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["gate"], x["beta"], cu_seqlens=cu,
                             chunk=32, fusion=fusion)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    o_ref, s_ref = _oracle_fused(x, fusion, None, cu.cpu().numpy())
    assert rel_err(o.reshape(-1, H, Dv), o_ref) <= TOL_F32
    assert rel_err(s, s_ref) <= TOL_F32


@pytest.mark.parametrize("dtype,dims", [("bf16", (128, 128)), ("f32", (40, 12))])
@pytest.mark.parametrize("T", [9, 37])
def test_recurrent_fused(cuda_device, dtype, dims, T):
    Dk, Dv = dims
    N, H = 4, 3
    x = _raw_inputs(N, T, H, Dk, Dv, dtype, 720, cuda_device)
    fusion = dict(qk_l2norm=True, eps=1e-6, A_log=x["A_log"], dt_bias=x["dt_bias"])
    pool = torch.randn((N, H, Dk, Dv), device=cuda_device) * 0.05
    pool0 = pool.clone()
    o = kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["gate"], x["beta"], pool, fusion=fusion)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    o_ref, s_ref = _oracle_fused(x, fusion, pool0.cpu(), np.arange(N + 1) * T)
    tol_o = TOL_DECODE_O if dtype == "bf16" else TOL_F32
    assert rel_err(o.reshape(-1, H, Dv), o_ref) <= tol_o
    assert rel_err(pool, s_ref) <= TOL_DECODE_S


def test_fused_without_options_equals_plain_call(cuda_device):
    x = _raw_inputs(1, 130, 2, 128, 128, "bf16", 730, cuda_device)
    la = -torch.nn.functional.softplus(x["gate"]) * 0.5
    k = (x["k"].float() / x["k"].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    a, sa = kda.kda_chunk_fwd(x["q"], k, x["v"], la, x["beta"], chunk=64)
    b, sb = kda.kda_chunk_fwd(x["q"], k, x["v"], la, x["beta"], chunk=64, fusion={})
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(sa, sb)
