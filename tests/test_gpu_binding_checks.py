"""The binding refuses, before anything is launched, buffers a call would write out of bounds or
read from the wrong memory: mis-shaped or mis-typed outputs, host tensors, a host workspace, and
inputs whose shapes disagree with q. A workspace is counted in bytes whatever its dtype."""
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth

pytestmark = [pytest.mark.gpu, pytest.mark.late]


def _prefill_args(dev):
    spec = kda_synth.PrefillSpec("t", B=1, T=64, H=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                                 decay="fast", init_std=0.0)
    x = kda_synth.prefill_inputs(spec, 5, dev)
    return [x[n] for n in ("q", "k", "v", "log_alpha", "beta")]


def test_prefill_outputs_and_workspace_are_checked(cuda_device):
    args = _prefill_args(cuda_device)
    bf = dict(dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(ValueError):  # one token short
        kda.kda_chunk_fwd(*args, o=torch.empty((1, 63, 2, 128), **bf))
    with pytest.raises(TypeError):  # o in another dtype than q
        kda.kda_chunk_fwd(*args, o=torch.empty((1, 64, 2, 128), dtype=torch.float32,
                                               device=cuda_device))
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(*args, final_state=torch.empty((1, 2, 128, 64), device=cuda_device))
    with pytest.raises(ValueError):  # a workspace in host memory
        kda.kda_chunk_fwd(*args, workspace=torch.empty(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError):  # host q on the no-allocation entry point
        kda.kda_chunk_fwd_noalloc(args[0].cpu(), *args[1:])
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd_noalloc(*args, o=torch.empty((1, 64, 2, 64), **bf))
    # an fp32 workspace of enough bytes is used as it is
    nbytes = kda.kda_chunk_fwd_workspace_size(1, 64, 2, 128, 128, 64, 1, torch.bfloat16)
    ws = torch.zeros((nbytes + 3) // 4, dtype=torch.float32, device=cuda_device)
    o, s = kda.kda_chunk_fwd(*args, workspace=ws)
    o2, s2 = kda.kda_chunk_fwd(*args)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.equal(o, o2) and torch.equal(s, s2)


def test_decode_and_recurrent_shapes_are_checked(cuda_device):
    N, H, d, T = 4, 2, 128, 3
    g = torch.Generator(device=cuda_device).manual_seed(3)
    bf = dict(dtype=torch.bfloat16, device=cuda_device)
    q = torch.randn((N, H, d), generator=g, device=cuda_device).to(torch.bfloat16)
    la = -torch.rand((N, H, d), generator=g, device=cuda_device)
    beta = torch.rand((N, H), generator=g, device=cuda_device)
    state = torch.zeros((N, H, d, d), device=cuda_device)
    with pytest.raises(ValueError):
        kda.kda_recurrent_step(q, q, q, la, beta, state, o=torch.empty((N, H, d - 4), **bf))
    with pytest.raises(ValueError):  # beta of another shape
        kda.kda_recurrent_step(q, q, q, la, beta[:, :1].contiguous(), state)
    with pytest.raises(ValueError):  # v for fewer sequences
        kda.kda_recurrent_step(q, q, q[:2].contiguous(), la, beta, state)
    qT = torch.randn((N, T, H, d), generator=g, device=cuda_device).to(torch.bfloat16)
    laT = -torch.rand((N, T, H, d), generator=g, device=cuda_device)
    bT = torch.rand((N, T, H), generator=g, device=cuda_device)
    pool = torch.zeros((N, H, d, d), device=cuda_device)
    with pytest.raises(ValueError):
        kda.kda_recurrent_fwd(qT, qT, qT, laT, bT, pool, o=torch.empty((N, T + 1, H, d), **bf))
    with pytest.raises(ValueError):
        kda.kda_recurrent_fwd(qT, qT, qT, laT, bT[:, :, :1].contiguous(), pool)
    torch.cuda.synchronize()
    assert not state.any() and not pool.any()  # nothing was launched
