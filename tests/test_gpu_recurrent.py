"""GPU parity of kda_recurrent_fwd (token-by-token mode over short sequences, states from a pool)
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
import oracle
from tests._parity import TOL_DECODE_O, TOL_DECODE_S, TOL_F32, rel_err, to_np

pytestmark = pytest.mark.gpu


def _inputs(N, T, H, Dk, Dv, dtype, seed, dev):
    spec = kda_synth.PrefillSpec("r", B=N, T=T, H=H, Dk=Dk, Dv=Dv, chunk=64, dtype=dtype,
                                 decay="fast", init_std=0.0)
    return kda_synth.prefill_inputs(spec, seed, dev)


@pytest.mark.parametrize("dtype,dims", [("bf16", (128, 128)), ("f32", (40, 12)),
                                        ("bf16", (64, 128)), ("f32", (128, 128))])
@pytest.mark.parametrize("T", [1, 2, 7, 16, 37, 64])
def test_recurrent_fwd_with_state_pool(cuda_device, dtype, dims, T):
    Dk, Dv = dims
    N, H, P = 6, 3, 10
    x = _inputs(N, T, H, Dk, Dv, dtype, 600 + T + Dk, cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(7)
    pool = torch.randn((P, H, Dk, Dv), generator=g, device=cuda_device) * 0.05
    idx = torch.tensor([7, 2, -1, 0, 9, 4], dtype=torch.int32, device=cuda_device)
    pool0 = pool.clone()
    o = torch.full((N, T, H, Dv), 3.0, dtype=x["q"].dtype, device=cuda_device)
    kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, idx, o=o)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    live = [n for n in range(N) if int(idx[n]) >= 0]
    slots = [int(idx[n]) for n in live]
    sub = {n_: x[n_][live].cpu() for n_ in ("q", "k", "v", "log_alpha", "beta")}
    cu = np.arange(len(live) + 1, dtype=np.int64) * T
    o_ref, s_ref = oracle.recurrent(sub["q"].reshape(-1, H, Dk), sub["k"].reshape(-1, H, Dk),
                                    sub["v"].reshape(-1, H, Dv),
                                    sub["log_alpha"].reshape(-1, H, Dk),
                                    sub["beta"].reshape(-1, H),
                                    initial_state=pool0[slots].cpu(), cu_seqlens=cu)
    tol_o = TOL_DECODE_O if dtype == "bf16" else TOL_F32
    assert rel_err(o[live].reshape(-1, H, Dv), o_ref) <= tol_o
    assert rel_err(pool[slots], s_ref) <= TOL_DECODE_S
    untouched = [p for p in range(P) if p not in slots]
    assert torch.equal(pool[untouched], pool0[untouched])
    assert torch.all(o[2] == 3.0)  # the skipped sequence's output is left alone


def test_recurrent_fwd_matches_chunked_prefill(cuda_device):
    """The recurrent mode and the chunkwise mode are two evaluations of the same operator."""
    N, T, H = 2, 64, 4
    x = _inputs(N, T, H, 128, 128, "bf16", 650, cuda_device)
    s0 = torch.randn((N, H, 128, 128), device=cuda_device) * 0.02
    pool = s0.clone()
    o_rec = kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool)
    o_chk, s_chk = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                     initial_state=s0, chunk=64)
    torch.cuda.synchronize()
    assert rel_err(o_rec, to_np(o_chk)) <= 2e-2
    assert rel_err(pool, to_np(s_chk)) <= 2e-2


def test_recurrent_fwd_index_beyond_pool_is_reported(cuda_device):
    N, T, H = 3, 4, 2
    x = _inputs(N, T, H, 32, 32, "f32", 660, cuda_device)
    pool = torch.zeros((2, H, 32, 32), device=cuda_device)
    idx = torch.tensor([0, 5, 1], dtype=torch.int32, device=cuda_device)
    kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, idx)
    assert kda.kda_last_device_error() == kda.KDA_ERR_INVALID_ARG
    assert torch.isfinite(pool).all()
    assert kda.kda_last_device_error() == kda.KDA_OK


def test_recurrent_fwd_strong_and_mild_decays_in_one_launch(cuda_device):
    """Items whose decay over the call stays mild and items whose channels decay by hundreds of
    nats within the call in one launch (the chunk-form kernel factors the first kind's ratios
    around each channel's midpoint and forms the second kind's exactly), against the oracle at
    the recurrent mode's tolerances."""
    N, T, H = 8, 12, 3
    x = _inputs(N, T, H, 128, 128, "bf16", 670, cuda_device)
    la = x["log_alpha"].clone()
    la[1::2] *= 25.0  # odd sequences: about -40 per token on average over 12 tokens
    x["log_alpha"] = la
    g = torch.Generator(device=cuda_device).manual_seed(71)
    pool = torch.randn((N, H, 128, 128), generator=g, device=cuda_device) * 0.05
    pool0 = pool.clone()
    o = kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    cu = np.arange(N + 1, dtype=np.int64) * T
    o_ref, s_ref = oracle.recurrent(*(x[n_].cpu().reshape(N * T, H, -1) if n_ != "beta"
                                      else x[n_].cpu().reshape(N * T, H)
                                      for n_ in ("q", "k", "v", "log_alpha", "beta")),
                                    initial_state=pool0.cpu(), cu_seqlens=cu)
    assert torch.isfinite(pool).all()
    assert rel_err(o.reshape(-1, H, 128), o_ref) <= TOL_DECODE_O
    assert rel_err(pool, s_ref) <= TOL_DECODE_S

