"""Deterministic replay, the substitute for a race detector: the same inputs twice give
bit-identical outputs (no kernel reduces through atomics, so every sum has one order). Covers the
paths the other replay tests do not: the multi-token recurrent mode with pooled states, the
prefill with the fused prologue and output epilogue (two-CTA clusters exchanging row sums), and a
packed varlen batch (state chains in longest-first order)."""
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth

pytestmark = [pytest.mark.gpu, pytest.mark.late]


def test_recurrent_mode_replays_bit_exactly(cuda_device):
    N, T, H, d = 8, 16, 4, 128
    spec = kda_synth.PrefillSpec("r", B=N, T=T, H=H, Dk=d, Dv=d, chunk=64, dtype="bf16",
                                 decay="slow", init_std=0.0)
    x = kda_synth.prefill_inputs(spec, 1500, cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(1501)
    pool0 = torch.randn((2 * N, H, d, d), generator=g, device=cuda_device) * 0.02
    idx = torch.randperm(2 * N, generator=g, device=cuda_device)[:N].to(torch.int32)
    runs = []
    for _ in range(2):
        pool = pool0.clone()
        o = kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, idx)
        runs.append((o, pool))
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])


def test_fused_layer_prefill_replays_bit_exactly(cuda_device):
    B, T, H, d = 2, 300, 4, 128
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(1510)
    q = (torch.randn((B, T, H, d), generator=g, device=dev) * 3).to(torch.bfloat16)
    k = (torch.randn((B, T, H, d), generator=g, device=dev) * 3).to(torch.bfloat16)
    v = torch.randn((B, T, H, d), generator=g, device=dev).to(torch.bfloat16)
    gate = torch.randn((B, T, H, d), generator=g, device=dev) - 1.0
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, device=dev))
    fusion = dict(qk_l2norm=True, eps=1e-6,
                  A_log=torch.log(torch.rand((H,), generator=g, device=dev) * 15 + 1) - 2.0,
                  dt_bias=torch.randn((H, d), generator=g, device=dev) * 0.5,
                  out_norm=True, out_norm_eps=1e-5,
                  out_norm_weight=torch.rand((d,), generator=g, device=dev) + 0.5,
                  out_gate=torch.randn((B, T, H, d), generator=g, device=dev).to(torch.bfloat16))
    s0 = torch.randn((B, H, d, d), generator=g, device=dev) * 0.02
    a, sa = kda.kda_chunk_fwd(q, k, v, gate, beta, initial_state=s0, fusion=fusion)
    b, sb = kda.kda_chunk_fwd(q, k, v, gate, beta, initial_state=s0, fusion=fusion)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.equal(a, b) and torch.equal(sa, sb)


def test_varlen_prefill_replays_bit_exactly(cuda_device):
    spec = kda_synth.varlen_spec(1520, n=12, lo=64, hi=2048)
    x = kda_synth.prefill_inputs(spec, 1521, cuda_device)
    runs = [kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                              cu_seqlens=x["cu_seqlens"], chunk=64) for _ in range(2)]
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])
