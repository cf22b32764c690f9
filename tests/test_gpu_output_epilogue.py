"""GPU parity of the output epilogue (head-wise RMSNorm x sigmoid gate applied to the operator's
output before the store) on the chunkwise (bf16 cluster path, fp32 pass) and recurrent paths,
against the fp64 oracle's recurrence followed by its output_norm_gate."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
import oracle
from kda_synth import PrefillSpec
from tests._parity import TOL_BF16_O, TOL_DECODE_O, TOL_F32, rel_err, to_np

pytestmark = pytest.mark.gpu


def _epilogue(dev, shape, dtype, seed, gate=True, weight=True):
    g = torch.Generator(device=dev).manual_seed(seed)
    Dv = shape[-1]
    w = (torch.rand((Dv,), generator=g, device=dev) * 1.5 + 0.25) if weight else None
    og = (torch.randn(shape, generator=g, device=dev) * 2.0).to(dtype) if gate else None
    return dict(out_norm=True, out_norm_eps=1e-5, out_norm_weight=w, out_gate=og)


def _gate_weight(fz, H, Dv, rows):
    gate = None if fz["out_gate"] is None else to_np(fz["out_gate"]).reshape(-1, H, Dv)[:rows]
    w = None if fz["out_norm_weight"] is None else to_np(fz["out_norm_weight"])
    return gate, w


def _oracle_y(inp, fz, cu, H):
    """(y_ref, final_state_ref, o_ref): the oracle's recurrence, then its epilogue."""
    o, s = oracle.recurrent(*(inp[x].cpu() for x in ("q", "k", "v", "log_alpha", "beta")),
                            initial_state=None if inp.get("initial_state") is None
                            else inp["initial_state"].cpu(), cu_seqlens=cu)
    gate, w = _gate_weight(fz, H, o.shape[-1], o.shape[0])
    return oracle.output_norm_gate(o, gate, w, fz["out_norm_eps"]), s, o


def epilogue_err(y, y_ref, o_ref, fz, H):
    """Error of y in the units of the operator's output: the normalisation divides each row by its
    own RMS, so a row with a small o carries o's absolute error magnified; undoing it row by row
    (times the row's RMS, divided by weight x sigmoid(gate)) gives the error of the underlying o
    relative to max|o|, the quantity the output tolerance bounds."""
    Dv = o_ref.shape[-1]
    y = to_np(y).reshape(o_ref.shape)
    gate, w = _gate_weight(fz, H, Dv, o_ref.shape[0])
    scale = np.sqrt(np.mean(o_ref * o_ref, axis=-1, keepdims=True) + fz["out_norm_eps"])
    scale = scale / (1.0 if w is None else w) / (1.0 if gate is None else oracle._sigmoid(gate))
    return np.abs((y - y_ref) * scale).max() / np.abs(o_ref).max()


@pytest.mark.parametrize("T", [200, 4096])
def test_chunk_bf16_output_epilogue(cuda_device, T):
    """Clusters of two CTAs exchange the row sums of squares of their column halves; T = 4096
    runs 64 chunks through the exchange's double-buffered barriers."""
    B, H = 2, 3
    spec = PrefillSpec("t", B=B, T=T, H=H, Dk=128, Dv=128, chunk=64, dtype="bf16",
                       decay="fast", init_std=0.02)
    inp = kda_synth.prefill_inputs(spec, 800 + T, cuda_device)
    fz = _epilogue(cuda_device, inp["v"].shape, torch.bfloat16, 801)
    y, s = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             initial_state=inp["initial_state"], chunk=64, fusion=fz)
    o_plain, s_plain = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                         inp["beta"], initial_state=inp["initial_state"], chunk=64)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.equal(s, s_plain)  # the epilogue touches the output only
    y_ref, _, o_ref = _oracle_y(inp, fz, np.arange(B + 1) * T, H)
    assert epilogue_err(y, y_ref, o_ref, fz, H) <= TOL_BF16_O
    # the same epilogue applied by the oracle to the GPU's own plain output: they differ only by
    # the bf16 rounding of o before the normalisation
    y_from_plain = oracle.output_norm_gate(to_np(o_plain), to_np(fz["out_gate"]),
                                           to_np(fz["out_norm_weight"]), 1e-5)
    assert rel_err(y, y_from_plain) <= 1e-2


@pytest.mark.parametrize("gated", [False, True], ids=["no_gate", "gate_and_weight"])
def test_chunk_bf16_output_epilogue_varlen(cuda_device, gated):
    """Packed sequences with ragged last chunks: the gate rows of a chunk's padding rows belong to
    the next sequence (or lie past the batch) and must not be read into the output."""
    lens = [130, 0, 64, 1, 257]
    T = sum(lens)
    spec = PrefillSpec("t", B=1, T=T, H=2, Dk=128, Dv=128, chunk=64, dtype="bf16", decay="fast",
                       init_std=0.0, seqlens=tuple(lens))
    inp = kda_synth.prefill_inputs(spec, 810, cuda_device)
    fz = _epilogue(cuda_device, inp["v"].shape, torch.bfloat16, 811, gate=gated, weight=gated)
    y, _ = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             cu_seqlens=inp["cu_seqlens"], chunk=64, fusion=fz)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    y_ref, _, o_ref = _oracle_y(inp, fz, inp["cu_seqlens"].cpu().numpy(), 2)
    assert epilogue_err(y, y_ref, o_ref, fz, 2) <= TOL_BF16_O
    if gated:
        return
    # ungated, unweighted rows have RMS sqrt(ms / (ms + eps)) for the mean square ms of o: ~1 for
    # every row well above eps
    ms = np.mean(o_ref * o_ref, axis=-1)
    rms = to_np(y.float().pow(2).mean(-1).sqrt()).reshape(ms.shape)
    big = ms > 100 * 1e-5
    assert big.mean() > 0.5
    assert np.abs(rms[big] - 1.0).max() <= 2e-2


def test_chunk_f32_output_epilogue_varlen(cuda_device):
    """The fp32 path applies the epilogue as its own pass; tokens past the last sequence end
    are left alone."""
    lens = [5, 70, 0, 33]
    T, H, Dk, Dv = sum(lens) + 6, 2, 48, 20
    spec = PrefillSpec("t", B=1, T=T, H=H, Dk=Dk, Dv=Dv, chunk=32, dtype="f32", decay="fast",
                       init_std=0.0)
    inp = kda_synth.prefill_inputs(spec, 820, cuda_device)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32,
                      device=cuda_device)
    fz = _epilogue(cuda_device, inp["v"].shape, torch.float32, 821)
    o = torch.full_like(inp["v"], 7.0)
    kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], cu_seqlens=cu,
                      chunk=32, o=o, fusion=fz)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    n = int(cu[-1])
    sub = {x: inp[x][:, :n] for x in ("q", "k", "v", "log_alpha", "beta")}
    fz_sub = dict(fz, out_gate=fz["out_gate"][:, :n])
    y_ref, _, o_ref = _oracle_y(sub, fz_sub, cu.cpu().numpy(), H)
    assert epilogue_err(o[:, :n], y_ref, o_ref, fz_sub, H) <= TOL_F32
    assert torch.all(o[:, n:] == 7.0)


@pytest.mark.parametrize("dtype,dims", [("bf16", (128, 128)), ("f32", (40, 12))])
@pytest.mark.parametrize("T", [9, 37])
def test_recurrent_output_epilogue(cuda_device, dtype, dims, T):
    """T = 37 runs three chunks of the chunk-form kernel (d = 128), the last one ragged."""
    Dk, Dv = dims
    N, H = 4, 3
    spec = PrefillSpec("r", B=N, T=T, H=H, Dk=Dk, Dv=Dv, chunk=64, dtype=dtype, decay="fast",
                       init_std=0.0)
    inp = kda_synth.prefill_inputs(spec, 830, cuda_device)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    fz = _epilogue(cuda_device, inp["v"].shape, tdt, 831)
    pool = torch.randn((N, H, Dk, Dv), device=cuda_device) * 0.05
    pool0 = pool.clone()
    y = kda.kda_recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], pool,
                              fusion=fz)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    inp["initial_state"] = pool0
    y_ref, s_ref, o_ref = _oracle_y(inp, fz, np.arange(N + 1) * T, H)
    tol = TOL_DECODE_O if dtype == "bf16" else TOL_F32
    assert epilogue_err(y, y_ref, o_ref, fz, H) <= tol
    assert rel_err(pool, s_ref) <= 1e-4


def test_prologue_and_epilogue_together(cuda_device):
    """Raw q, k and gates in, normalised gated output out: the whole fused layer core."""
    B, T, H = 1, 1000, 4
    g = torch.Generator(device=cuda_device).manual_seed(840)
    q = (torch.randn((B, T, H, 128), generator=g, device=cuda_device) * 3).to(torch.bfloat16)
    k = (torch.randn((B, T, H, 128), generator=g, device=cuda_device) * 3).to(torch.bfloat16)
    v = torch.randn((B, T, H, 128), generator=g, device=cuda_device).to(torch.bfloat16)
    gate = torch.randn((B, T, H, 128), generator=g, device=cuda_device) - 1.0
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, device=cuda_device))
    A_log = torch.log(torch.rand((H,), generator=g, device=cuda_device) * 15 + 1) - 2.0
    dt_bias = torch.randn((H, 128), generator=g, device=cuda_device) * 0.5
    fz = _epilogue(cuda_device, v.shape, torch.bfloat16, 841)
    fz.update(qk_l2norm=True, eps=1e-6, A_log=A_log, dt_bias=dt_bias)
    y, s = kda.kda_chunk_fwd(q, k, v, gate, beta, chunk=64, fusion=fz)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    qn, kn, la = oracle.prologue(q.cpu(), k.cpu(), gate.cpu(), A_log=A_log.cpu(),
                                 dt_bias=dt_bias.cpu(), qk_l2norm=True, eps=1e-6)
    o_ref, s_ref = oracle.recurrent(qn.reshape(-1, H, 128), kn.reshape(-1, H, 128), v.cpu(),
                                    la.reshape(-1, H, 128), beta.cpu())
    y_ref = oracle.output_norm_gate(o_ref, to_np(fz["out_gate"]).reshape(-1, H, 128),
                                    to_np(fz["out_norm_weight"]), 1e-5)
    assert epilogue_err(y, y_ref, o_ref, fz, H) <= TOL_BF16_O
    assert rel_err(s, s_ref) <= 2e-2
