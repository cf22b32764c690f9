"""The library's calls captured in CUDA graphs and replayed.

A serving loop removes launch overhead by capturing its steps once and replaying the graph. The
compute entry points make no synchronising or allocating call while they run (given their
workspace), so a stream capture records exactly their kernel launches (the programmatic
dependent launch between the two prefill kernels included). These tests capture a decode loop, a
prefill call with a caller-owned workspace (fixed-length and packed varlen), the fused decode
step and the multi-token recurrent mode, replay each graph, and check the replay against the same
calls run eagerly: the kernels are deterministic, so the results must be identical.
"""
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
from kda_synth import DecodeSpec, PrefillSpec

pytestmark = [pytest.mark.gpu, pytest.mark.late]


def _capture(fn):
    """Warm `fn` up on a side stream (first-call set-up such as kernel attributes happens outside
    the capture), then capture one call of it into a graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_loop_replayed_from_a_graph(cuda_device):
    spec = DecodeSpec("d", N=32, H=4, Dk=128, Dv=128, steps=8, dtype="bf16", decay="slow",
                      init_std=0.02)
    s0 = kda_synth.decode_state(spec, 81, cuda_device)
    x = kda_synth.decode_step_inputs(spec, 81, spec.steps, cuda_device)
    state = s0.clone()
    outs = torch.empty((spec.steps, spec.N, spec.H, spec.Dv), dtype=torch.bfloat16,
                       device=cuda_device)

    def loop():
        for t in range(spec.steps):
            kda.kda_recurrent_step(x["q"][t], x["k"][t], x["v"][t], x["log_alpha"][t],
                                   x["beta"][t], state, o=outs[t])

    g = _capture(loop)
    # eager reference from the same initial state
    state.copy_(s0)
    loop()
    torch.cuda.synchronize()
    ref_o, ref_s = outs.clone(), state.clone()
    # replay twice from the initial state
    for _ in range(2):
        outs.zero_()
        state.copy_(s0)
        g.replay()
        torch.cuda.synchronize()
        assert kda.kda_last_device_error() == kda.KDA_OK
        assert torch.equal(outs, ref_o) and torch.equal(state, ref_s)


@pytest.mark.parametrize("varlen", [False, True], ids=["fixed_length", "packed_varlen"])
def test_prefill_replayed_from_a_graph(cuda_device, varlen):
    spec = (PrefillSpec("v", B=1, T=700, H=4, Dk=128, Dv=128, chunk=64, dtype="bf16",
                        decay="fast", init_std=0.0, seqlens=(1, 300, 0, 399)) if varlen else
            PrefillSpec("f", B=2, T=333, H=4, Dk=128, Dv=128, chunk=64, dtype="bf16",
                        decay="fast", init_std=0.02))
    x = kda_synth.prefill_inputs(spec, 82, cuda_device)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_size(spec.B, spec.T, spec.H, 128, 128, 64,
                                                      spec.num_seqs, torch.bfloat16),
                     dtype=torch.uint8, device=cuda_device)
    o = torch.empty_like(x["v"])
    fs = torch.empty((spec.num_seqs, spec.H, 128, 128), dtype=torch.float32, device=cuda_device)

    def call():
        kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                          initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                          chunk=64, o=o, final_state=fs, workspace=ws)

    g = _capture(call)
    call()
    torch.cuda.synchronize()
    ref_o, ref_s = o.clone(), fs.clone()
    o.zero_()
    fs.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.equal(o, ref_o) and torch.equal(fs, ref_s)


def test_fused_decode_and_recurrent_mode_replayed_from_graphs(cuda_device):
    dev = cuda_device
    gen = torch.Generator(device=dev).manual_seed(83)
    N, H, D = 8, 4, 128
    fusion = dict(qk_l2norm=True, eps=1e-6,
                  A_log=torch.randn((H,), generator=gen, device=dev),
                  dt_bias=torch.randn((H, D), generator=gen, device=dev) * 0.5,
                  out_norm=True, out_norm_eps=1e-5,
                  out_norm_weight=torch.rand((D,), generator=gen, device=dev) + 0.5,
                  out_gate=torch.randn((N, H, D), generator=gen, device=dev).to(torch.bfloat16))
    q = torch.randn((N, H, D), generator=gen, device=dev).to(torch.bfloat16)
    k = torch.randn((N, H, D), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((N, H, D), generator=gen, device=dev).to(torch.bfloat16)
    gate = torch.randn((N, H, D), generator=gen, device=dev) - 1.0
    beta = torch.sigmoid(torch.randn((N, H), generator=gen, device=dev))
    s0 = torch.randn((N, H, D, D), generator=gen, device=dev) * 0.05
    state = s0.clone()
    y = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)

    def step():
        kda.kda_recurrent_step(q, k, v, gate, beta, state, o=y, fusion=fusion)

    # the multi-token recurrent mode over a pool with a skipped slot
    rspec = PrefillSpec("r", B=6, T=9, H=H, Dk=D, Dv=D, chunk=64, dtype="bf16", decay="fast",
                        init_std=0.0)
    xr = kda_synth.prefill_inputs(rspec, 84, dev)
    p0 = torch.randn((8, H, D, D), generator=gen, device=dev) * 0.05
    pool = p0.clone()
    idx = torch.tensor([7, 2, -1, 0, 5, 4], dtype=torch.int32, device=dev)
    yr = torch.zeros_like(xr["v"])

    def rec():
        kda.kda_recurrent_fwd(xr["q"], xr["k"], xr["v"], xr["log_alpha"], xr["beta"], pool, idx,
                              o=yr)

    for fn, outs, st, st0 in ((step, y, state, s0), (rec, yr, pool, p0)):
        g = _capture(fn)
        st.copy_(st0)
        fn()
        torch.cuda.synchronize()
        ref_o, ref_s = outs.clone(), st.clone()
        outs.zero_()
        st.copy_(st0)
        g.replay()
        torch.cuda.synchronize()
        assert kda.kda_last_device_error() == kda.KDA_OK
        assert torch.equal(outs, ref_o) and torch.equal(st, ref_s)
