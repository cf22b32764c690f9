"""Guard canaries, a substitute for the memory checker (closed on this pool): every output, state
and workspace buffer handed to the library is the front of a larger allocation whose tail holds a
known pattern; after the call the tail must be untouched. Covers the tensor-core and fp32
prefill (ragged and packed with an empty sequence), the fused-layer prefill, the decode step,
the recurrent mode with a state pool and the backward pass's workspace."""
import math

import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth

pytestmark = [pytest.mark.gpu, pytest.mark.late]

GUARD = 4096  # guard elements after each buffer


def _guarded(shape, dtype, dev, fill):
    """(whole allocation, the contiguous front of `shape` the library may write)."""
    n = math.prod(shape)
    buf = torch.full((n + GUARD,), fill, dtype=dtype, device=dev)
    return buf, buf[:n].view(shape)


def _intact(buf, shape, fill):
    return bool(torch.all(buf[math.prod(shape):] == fill))


def _front(buf, shape, like):
    """The front of a guarded buffer, filled with `like`'s values (state inputs)."""
    front = buf[:math.prod(shape)].view(shape)
    front.copy_(like)
    return front


@pytest.mark.parametrize("path", ["bf16_ragged", "f32_packed", "bf16_fused_layer"])
def test_prefill_writes_stay_inside_their_buffers(cuda_device, path):
    dev = cuda_device
    fusion, cu = None, None
    if path == "f32_packed":
        lens = [5, 70, 0, 33]
        spec = kda_synth.PrefillSpec("t", B=1, T=sum(lens) + 6, H=2, Dk=48, Dv=20, chunk=32,
                                     dtype="f32", decay="fast", init_std=0.02)
        x = kda_synth.prefill_inputs(spec, 1600, dev)
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
        N = len(lens)
        s0 = torch.randn((N, 2, 48, 20), device=dev) * 0.02
    else:
        spec = kda_synth.PrefillSpec("t", B=2, T=150, H=2, Dk=128, Dv=128, chunk=64,
                                     dtype="bf16", decay="fast", init_std=0.02)
        x = kda_synth.prefill_inputs(spec, 1601, dev)
        N, s0 = 2, x["initial_state"]
        if path == "bf16_fused_layer":
            g = torch.Generator(device=dev).manual_seed(1602)
            fusion = dict(qk_l2norm=True, eps=1e-6,
                          A_log=torch.log(torch.rand((2,), generator=g, device=dev) * 15 + 1) - 2,
                          dt_bias=torch.randn((2, 128), generator=g, device=dev) * 0.5,
                          out_norm=True, out_norm_eps=1e-5,
                          out_norm_weight=torch.rand((128,), generator=g, device=dev) + 0.5,
                          out_gate=torch.randn(x["v"].shape, generator=g,
                                               device=dev).to(x["v"].dtype))
    dt = x["q"].dtype
    o_shape = tuple(x["v"].shape)
    s_shape = (N, spec.H, spec.Dk, spec.Dv)
    o_buf, o = _guarded(o_shape, dt, dev, 7.0)
    s_buf, st = _guarded(s_shape, torch.float32, dev, 12345.0)
    nbytes = kda.kda_chunk_fwd_workspace_size(spec.B, spec.T, spec.H, spec.Dk, spec.Dv,
                                              spec.chunk, N, dt)
    w_buf = torch.full((nbytes + GUARD,), 0xA5, dtype=torch.uint8, device=dev)
    kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], initial_state=s0,
                      cu_seqlens=cu, chunk=spec.chunk, o=o, final_state=st,
                      workspace=w_buf[:nbytes], fusion=fusion)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert _intact(o_buf, o_shape, 7.0) and _intact(s_buf, s_shape, 12345.0)
    assert bool(torch.all(w_buf[nbytes:] == 0xA5))
    if cu is not None:  # tokens past the last sequence are not written either
        assert bool(torch.all(o[:, int(cu[-1]):] == 7.0))


def test_decode_and_recurrent_writes_stay_inside_their_buffers(cuda_device):
    dev = cuda_device
    N, H, d, T = 6, 2, 128, 5
    spec = kda_synth.DecodeSpec("d", N=N, H=H, Dk=d, Dv=d, steps=1, dtype="bf16", decay="slow",
                                init_std=0.02)
    x = kda_synth.decode_step_inputs(spec, 1610, 1, dev)
    s_shape, o_shape = (N, H, d, d), (N, H, d)
    s_buf = torch.full((math.prod(s_shape) + GUARD,), 12345.0, device=dev)
    state = _front(s_buf, s_shape, kda_synth.decode_state(spec, 1610, dev))
    o_buf, o = _guarded(o_shape, torch.bfloat16, dev, 7.0)
    kda.kda_recurrent_step(x["q"][0], x["k"][0], x["v"][0], x["log_alpha"][0], x["beta"][0],
                           state, o=o)
    # recurrent mode: 5 tokens per sequence against a pool of 2N states, every other slot used
    rspec = kda_synth.PrefillSpec("r", B=N, T=T, H=H, Dk=d, Dv=d, chunk=64, dtype="bf16",
                                  decay="slow", init_std=0.0)
    r = kda_synth.prefill_inputs(rspec, 1611, dev)
    p_shape, ro_shape = (2 * N, H, d, d), (N, T, H, d)
    p_buf = torch.full((math.prod(p_shape) + GUARD,), 12345.0, device=dev)
    pool = _front(p_buf, p_shape, torch.randn(p_shape, device=dev) * 0.02)
    idx = torch.arange(0, 2 * N, 2, dtype=torch.int32, device=dev)
    ro_buf, ro = _guarded(ro_shape, torch.bfloat16, dev, 7.0)
    kda.kda_recurrent_fwd(r["q"], r["k"], r["v"], r["log_alpha"], r["beta"], pool, idx, o=ro)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert _intact(s_buf, s_shape, 12345.0) and _intact(o_buf, o_shape, 7.0)
    assert _intact(p_buf, p_shape, 12345.0) and _intact(ro_buf, ro_shape, 7.0)


def test_backward_workspace_writes_stay_inside(cuda_device):
    dev = cuda_device
    spec = kda_synth.PrefillSpec("t", B=1, T=150, H=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                                 decay="fast", init_std=0.02)
    x = kda_synth.prefill_inputs(spec, 1620, dev)
    d_o = torch.randn(x["v"].shape, device=dev).to(x["v"].dtype)
    nbytes = kda.kda_chunk_bwd_workspace_size(1, 150, 2, 128, 128, 1, torch.bfloat16)
    w_buf = torch.full((nbytes + GUARD,), 0xA5, dtype=torch.uint8, device=dev)
    kda.kda_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                      initial_state=x["initial_state"], workspace=w_buf[:nbytes])
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert bool(torch.all(w_buf[nbytes:] == 0xA5))
