"""GPU parity on the operator's degenerate inputs, on every path (bf16 tensor-core prefill, fp32
prefill, single-token decode, multi-token recurrent mode), against the fp64 oracle:
  - beta = 0 and log alpha = 0: nothing is written and nothing decays, so the state comes back
    bit for bit and o_t = S_0^T q_t;
  - beta = 0 with decay: the state only decays, S_T = Diag(prod alpha) S_0;
  - k = 0: no write reaches the state (its decay still applies);
  - log alpha = -30 per token: the state is forgotten at every token (the A matrices take the
    exact path on the tensor-core prefill);
  - v = 0 and S_0 = 0: every output and state is exactly zero."""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
import oracle
from tests._parity import (TOL_BF16_O, TOL_BF16_S, TOL_DECODE_O, TOL_DECODE_S, TOL_F32,
                           rel_err)

pytestmark = pytest.mark.gpu

CASES = ["frozen", "decay_only", "zero_keys", "total_decay", "all_zero"]
# (dtype, d, chunk) of the two prefill paths
PREFILL_PATHS = [("bf16", 128, 64), ("f32", 32, 32)]


def _degenerate(x, case):
    x = dict(x)
    if case in ("frozen", "decay_only"):
        x["beta"] = torch.zeros_like(x["beta"])
    if case == "frozen":
        x["log_alpha"] = torch.zeros_like(x["log_alpha"])
    if case == "zero_keys":
        x["k"] = torch.zeros_like(x["k"])
    if case == "total_decay":
        x["log_alpha"] = torch.full_like(x["log_alpha"], -30.0)
    if case == "all_zero":
        x["v"] = torch.zeros_like(x["v"])
    return x


@pytest.mark.parametrize("path", PREFILL_PATHS, ids=["bf16_tc", "f32"])
@pytest.mark.parametrize("case", CASES)
def test_prefill_degenerate(cuda_device, path, case):
    dtype, d, C = path
    B, T, H = 2, 150, 2
    spec = kda_synth.PrefillSpec("t", B=B, T=T, H=H, Dk=d, Dv=d, chunk=C, dtype=dtype,
                                 decay="fast", init_std=0.0 if case == "all_zero" else 0.05)
    x = _degenerate(kda_synth.prefill_inputs(spec, 1200 + CASES.index(case), cuda_device), case)
    s0 = x["initial_state"]
    o, s = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                             initial_state=s0, chunk=C)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(s).all()
    if case == "all_zero":
        assert not o.float().any() and not s.any()
        return
    if case == "frozen":
        assert torch.equal(s, s0)
    o_ref, s_ref = oracle.recurrent(*(x[n].cpu() for n in ("q", "k", "v", "log_alpha", "beta")),
                                    initial_state=None if s0 is None else s0.cpu(),
                                    cu_seqlens=np.arange(B + 1) * T)
    tol_o, tol_s = (TOL_BF16_O, TOL_BF16_S) if dtype == "bf16" else (TOL_F32, TOL_F32)
    assert rel_err(o.reshape(-1, H, d), o_ref) <= tol_o
    assert rel_err(s, s_ref) <= tol_s


@pytest.mark.parametrize("case", CASES)
def test_decode_and_recurrent_degenerate(cuda_device, case):
    """The same cases through kda_recurrent_step (one token) and kda_recurrent_fwd (T = 9, states
    from a pool)."""
    N, T, H, d = 4, 9, 2, 128
    spec = kda_synth.PrefillSpec("r", B=N, T=T, H=H, Dk=d, Dv=d, chunk=64, dtype="bf16",
                                 decay="fast", init_std=0.0)
    x = _degenerate(kda_synth.prefill_inputs(spec, 1300 + CASES.index(case), cuda_device), case)
    g = torch.Generator(device=cuda_device).manual_seed(1301)
    s0 = torch.zeros((N, H, d, d), device=cuda_device) if case == "all_zero" else \
        torch.randn((N, H, d, d), generator=g, device=cuda_device) * 0.05
    # decode: the first token of every sequence
    st = s0.clone()
    first = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    o1 = kda.kda_recurrent_step(first["q"], first["k"], first["v"], first["log_alpha"],
                                first["beta"], st)
    # recurrent mode: all T tokens
    pool = s0.clone()
    oT = kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    for o, s in ((o1, st), (oT, pool)):
        assert torch.isfinite(o.float()).all() and torch.isfinite(s).all()
    if case == "all_zero":
        assert not o1.float().any() and not st.any() and not oT.float().any() and not pool.any()
        return
    if case == "frozen":
        assert torch.equal(st, s0) and torch.equal(pool, s0)
    for tt, o, s in ((1, o1, st), (T, oT, pool)):
        sub = {n: x[n][:, :tt].cpu() for n in ("q", "k", "v", "log_alpha", "beta")}
        o_ref, s_ref = oracle.recurrent(*(sub[n].reshape(N * tt, H, -1) if n != "beta"
                                          else sub[n].reshape(N * tt, H)
                                          for n in ("q", "k", "v", "log_alpha", "beta")),
                                        initial_state=s0.cpu(),
                                        cu_seqlens=np.arange(N + 1) * tt)
        assert rel_err(o.reshape(N * tt, H, d), o_ref) <= TOL_DECODE_O
        assert rel_err(s, s_ref) <= TOL_DECODE_S
