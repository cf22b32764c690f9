"""kda_chunk_fwd_noalloc: prefill for callers that cannot allocate device scratch.

Some callers cannot give the library a workspace — a serving engine that has reserved almost all
of HBM for its caches, a plugin whose host framework owns every device allocation, or a loop that
must avoid cudaMalloc/cudaFree because they can stall the whole device. For them the library
keeps a fixed scratch array in its own device image. These tests call that entry point through
the C ABI and check that two calls in a row give what the workspace entry point gives, and that a
call needing more scratch than the array holds is refused before anything runs.

This file is collected last on purpose, so that a run which stops at its first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
from kda_synth import PrefillSpec
from tests._parity import TOL_BF16_O, TOL_BF16_S, TOL_F32, rel_err

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_abi(inp, spec, dt_code):
    """Call kda_chunk_fwd_noalloc directly through ctypes with caller-owned outputs."""
    dev = inp["q"].device
    o = torch.empty_like(inp["v"])
    fs = torch.empty((spec.num_seqs, spec.H, spec.Dk, spec.Dv), dtype=torch.float32, device=dev)
    rc = kda.lib().kda_chunk_fwd_noalloc(
        _p(inp["q"]), _p(inp["k"]), _p(inp["v"]), dt_code, _p(inp["log_alpha"]),
        _p(inp["beta"]), _p(inp["initial_state"]), _p(inp["cu_seqlens"]), spec.num_seqs,
        spec.B, spec.T, spec.H, spec.Dk, spec.Dv, spec.chunk, _p(o), _p(fs),
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    return rc, o, fs


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    cases = [
        (PrefillSpec("a", B=2, T=200, H=3, Dk=128, Dv=128, chunk=64, dtype="bf16",
                     decay="fast", init_std=0.02), kda.KDA_DTYPE_BF16, TOL_BF16_O, TOL_BF16_S),
        (PrefillSpec("b", B=1, T=108, H=2, Dk=32, Dv=16, chunk=32, dtype="f32", decay="fast",
                     init_std=0.02, seqlens=(5, 70, 0, 33)), kda.KDA_DTYPE_F32, TOL_F32,
         TOL_F32),
    ]
    for i, (spec, code, tol_o, tol_s) in enumerate(cases):
        inp = kda_synth.prefill_inputs(spec, 300 + i, cuda_device)
        o_ref, s_ref = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                         inp["beta"], initial_state=inp["initial_state"],
                                         cu_seqlens=inp["cu_seqlens"], chunk=spec.chunk)
        rc, o, s = _noalloc_abi(inp, spec, code)
        assert rc == kda.KDA_OK, kda.status_string(rc)
        torch.cuda.synchronize()
        assert kda.kda_last_device_error() == kda.KDA_OK
        assert rel_err(o, o_ref) <= tol_o
        assert rel_err(s, s_ref) <= tol_s


def test_noalloc_refuses_calls_beyond_its_scratch(cuda_device):
    # 256 chunks x 4 heads of records need more than the 64 MiB array: refused on the host
    spec = PrefillSpec("big", B=1, T=64 * 256, H=4, Dk=128, Dv=128, chunk=64, dtype="bf16",
                       decay="fast", init_std=0.0)
    need = kda.kda_chunk_fwd_workspace_size(spec.B, spec.T, spec.H, 128, 128, 64, 1,
                                            torch.bfloat16)
    assert need > kda.NOALLOC_SCRATCH_BYTES
    inp = kda_synth.prefill_inputs(spec, 400, cuda_device)
    rc, o, _ = _noalloc_abi(inp, spec, kda.KDA_DTYPE_BF16)
    assert rc == kda.KDA_ERR_WORKSPACE
