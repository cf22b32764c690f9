"""kda_chunk_fwd_noalloc: prefill for callers that cannot allocate device scratch.

Some callers cannot give the library a workspace — a serving engine that has reserved almost all
of HBM for its caches, a plugin whose host framework owns every device allocation, or a loop that
must avoid cudaMalloc/cudaFree because they can stall the whole device. For them the library
keeps a fixed scratch array in its own device image. These tests call that entry point through
the C ABI, twice in a row, and check each call against the workspace entry point (the same
kernels run, so the results must be identical, not only within the parity tolerance); they also
call it once through the Python wrapper with caller-owned outputs, and check that a call needing
more scratch than the array holds is refused before anything runs.

The tests are marked `late` and the file is named to sort last, so that it runs after every other
test: a run which stops at its first failure has then already run all the others.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
from kda_synth import PrefillSpec
from tests._parity import TOL_BF16_O, TOL_BF16_S, TOL_F32, rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.late]


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_abi(inp, spec, dt_code):
    """Call kda_chunk_fwd_noalloc directly through ctypes with caller-owned outputs."""
    dev = inp["q"].device
    o = torch.empty_like(inp["v"])
    fs = torch.empty((spec.num_seqs, spec.H, spec.Dk, spec.Dv), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = kda.lib().kda_chunk_fwd_noalloc(
            _p(inp["q"]), _p(inp["k"]), _p(inp["v"]), dt_code, _p(inp["log_alpha"]),
            _p(inp["beta"]), _p(inp["initial_state"]), _p(inp["cu_seqlens"]), spec.num_seqs,
            spec.B, spec.T, spec.H, spec.Dk, spec.Dv, spec.chunk, _p(o), _p(fs),
            ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    return rc, o, fs


CASES = [
    (PrefillSpec("a", B=2, T=200, H=3, Dk=128, Dv=128, chunk=64, dtype="bf16",
                 decay="fast", init_std=0.02), kda.KDA_DTYPE_BF16, TOL_BF16_O, TOL_BF16_S),
    (PrefillSpec("b", B=1, T=108, H=2, Dk=32, Dv=16, chunk=32, dtype="f32", decay="fast",
                 init_std=0.02, seqlens=(5, 70, 0, 33)), kda.KDA_DTYPE_F32, TOL_F32, TOL_F32),
]


@pytest.mark.parametrize("case", range(len(CASES)), ids=["bf16_tensor_cores", "f32_varlen"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device, case):
    spec, code, tol_o, tol_s = CASES[case]
    inp = kda_synth.prefill_inputs(spec, 300 + case, cuda_device)
    o_ref, s_ref = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                     initial_state=inp["initial_state"],
                                     cu_seqlens=inp["cu_seqlens"], chunk=spec.chunk)
    for call in range(2):  # the second call finds the first call's contents in the scratch array
        rc, o, s = _noalloc_abi(inp, spec, code)
        assert rc == kda.KDA_OK, kda.status_string(rc)
        torch.cuda.synchronize()
        assert kda.kda_last_device_error() == kda.KDA_OK
        assert rel_err(o, o_ref) <= tol_o and rel_err(s, s_ref) <= tol_s, call
        assert torch.equal(o, o_ref) and torch.equal(s, s_ref), call


def test_noalloc_python_wrapper_with_caller_outputs(cuda_device):
    spec, _, _, _ = CASES[0]
    inp = kda_synth.prefill_inputs(spec, 310, cuda_device)
    o_ref, s_ref = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                     initial_state=inp["initial_state"], chunk=64)
    o = torch.full_like(o_ref, float("nan"))
    fs = torch.full_like(s_ref, float("nan"))
    o2, s2 = kda.kda_chunk_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                       inp["beta"], initial_state=inp["initial_state"], chunk=64,
                                       o=o, final_state=fs)
    torch.cuda.synchronize()
    assert o2.data_ptr() == o.data_ptr() and s2.data_ptr() == fs.data_ptr()
    assert torch.equal(o, o_ref) and torch.equal(fs, s_ref)


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
