"""The bounds-checked build of the library (libkda_checked.so, compiled with KDA_BOUNDS_CHECK):
the kernels test their global accesses against the extent of the buffer each belongs to (the
tensor-core prefill, decode and recurrent-mode kernels access by access; the fp32 chunk kernels,
the output epilogue and the backward kernels by the first and last row of each work item), and an
access outside is skipped and reported through the status word instead of faulting. These tests
check that the check is really compiled in and fires (its self-test tests one access just past a
registered buffer, without performing it), that the normal build has none, and that the checked
build runs the operator's workloads with no report and with the normal build's results: the
tensor-core prefill (plain, packed varlen, fused), the decode step, the recurrent mode, the fp32
chunk kernels with the output epilogue, and the backward pass. The whole GPU suite can also run
on it: KDA_LIBRARY=<repo>/gated_delta_rule_120_b200/libkda_checked.so python -m pytest tests -m gpu.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

import gated_delta_rule_120_b200 as kda
from gated_delta_rule_120_b200 import _build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# run in a child process: the binding picks its library when it is first loaded
_CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["KDA_ROOT"])
import torch
import gated_delta_rule_120_b200 as kda
import kda_synth
from kda_synth import PrefillSpec
dev = torch.device("cuda:0")
out = {"lib": os.path.basename(kda.LIB_PATH)}
buf = torch.zeros(64, dtype=torch.uint8, device=dev)
out["selftest"] = int(kda.lib().kda_selftest_bounds(buf.data_ptr(), 64, None))
torch.cuda.synchronize()
out["selftest_status"] = kda.kda_last_device_error()
res = {}
for name, spec in (("bf16", PrefillSpec("a", B=2, T=300, H=3, Dk=128, Dv=128, chunk=64,
                                        dtype="bf16", decay="fast", init_std=0.02)),
                   ("varlen", PrefillSpec("b", B=1, T=400, H=2, Dk=128, Dv=128, chunk=64,
                                          dtype="bf16", decay="fast", init_std=0.0,
                                          seqlens=(1, 130, 0, 269)))):
    x = kda_synth.prefill_inputs(spec, 41, dev)
    o, s = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                             initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                             chunk=64)
    res[name] = (o, s)
g = torch.Generator(device=dev).manual_seed(5)
x = kda_synth.prefill_inputs(PrefillSpec("c", B=1, T=200, H=2, Dk=128, Dv=128, chunk=64,
                                         dtype="bf16", decay="fast", init_std=0.02), 43, dev)
fusion = dict(qk_l2norm=True, A_log=torch.randn(2, generator=g, device=dev),
              dt_bias=torch.randn(2, 128, generator=g, device=dev), out_norm=True,
              out_norm_weight=torch.rand(128, generator=g, device=dev) + 0.5,
              out_gate=torch.randn(x["v"].shape, generator=g, device=dev).to(torch.bfloat16))
res["fused"] = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                 initial_state=x["initial_state"], chunk=64, fusion=fusion)
dspec = kda_synth.DecodeSpec("d", N=16, H=4, Dk=128, Dv=128, steps=2, dtype="bf16",
                             decay="slow", init_std=0.02)
st = kda_synth.decode_state(dspec, 7, dev)
xs = kda_synth.decode_step_inputs(dspec, 7, 2, dev)
o = kda.kda_recurrent_step(xs["q"][0], xs["k"][0], xs["v"][0], xs["log_alpha"][0], xs["beta"][0], st)
res["decode"] = (o, st)
rspec = PrefillSpec("r", B=6, T=9, H=3, Dk=128, Dv=128, chunk=64, dtype="bf16", decay="fast",
                    init_std=0.0)
xr = kda_synth.prefill_inputs(rspec, 47, dev)
pool = torch.randn((8, 3, 128, 128), generator=g, device=dev) * 0.05
idx = torch.tensor([7, 2, -1, 0, 5, 4], dtype=torch.int32, device=dev)
# the skipped sequence (index -1) leaves its o rows untouched: start from zeros in both builds
o = kda.kda_recurrent_fwd(xr["q"], xr["k"], xr["v"], xr["log_alpha"], xr["beta"], pool, idx,
                          o=torch.zeros_like(xr["v"]))
res["recurrent"] = (o, pool)
# the fp32 path (CUDA-core chunk kernels) on a packed batch, with the output epilogue kernel
fspec = PrefillSpec("e", B=1, T=150, H=2, Dk=64, Dv=64, chunk=32, dtype="f32", decay="fast",
                    init_std=0.02, seqlens=(50, 0, 100))
xf = kda_synth.prefill_inputs(fspec, 44, dev)
res["f32_epilogue"] = kda.kda_chunk_fwd(
    xf["q"], xf["k"], xf["v"], xf["log_alpha"], xf["beta"], initial_state=xf["initial_state"],
    cu_seqlens=xf["cu_seqlens"], chunk=32,
    fusion=dict(out_norm=True, out_norm_weight=torch.rand(64, generator=g, device=dev) + 0.5,
                out_gate=torch.randn(xf["v"].shape, generator=g, device=dev)))
# the backward pass (bf16, and fp32 on the packed batch)
for name, bx in (("bwd_bf16", x), ("bwd_f32_varlen", xf)):
    d_o = torch.randn(bx["v"].shape, generator=g, device=dev).to(bx["v"].dtype)
    n_seq = bx["initial_state"].shape[0] if bx["initial_state"] is not None else \
        bx["cu_seqlens"].numel() - 1
    d_fin = torch.randn((n_seq,) + tuple(bx["v"].shape[2:3]) + (bx["q"].shape[-1], bx["v"].shape[-1]),
                        generator=g, device=dev)
    res[name] = kda.kda_chunk_bwd(bx["q"], bx["k"], bx["v"], bx["log_alpha"], bx["beta"], d_o,
                                  initial_state=bx["initial_state"], d_final_state=d_fin,
                                  cu_seqlens=bx["cu_seqlens"])
torch.cuda.synchronize()
out["status"] = kda.kda_last_device_error()
torch.save({k: tuple(t.float().cpu() for t in v if t is not None) for k, v in res.items()},
           os.environ["KDA_OUT"])
print(json.dumps(out))
"""


def _run_child(lib: str, out_path: str) -> dict:
    env = dict(os.environ, KDA_LIBRARY=lib, KDA_ROOT=ROOT, KDA_OUT=out_path)
    run = subprocess.run([sys.executable, "-c", _CHILD], env=env, capture_output=True, text=True,
                         timeout=600)
    assert run.returncode == 0, run.stdout[-2000:] + run.stderr[-2000:]
    return json.loads(run.stdout.strip().splitlines()[-1])


def test_checked_build_runs_the_workloads_clean_and_matches_the_normal_build(cuda_device,
                                                                            tmp_path):
    checked = _build.build(checked=True)
    normal = _build.build()
    a = _run_child(checked, str(tmp_path / "checked.pt"))
    b = _run_child(normal, str(tmp_path / "normal.pt"))
    assert a["lib"] == "libkda_checked.so" and b["lib"] == "libkda.so"
    # the check is compiled in and fires on an access past the registered extent ...
    assert a["selftest"] == kda.KDA_OK and a["selftest_status"] == kda.KDA_ERR_INVALID_ARG
    # ... and is absent from the normal build
    assert b["selftest"] == kda.KDA_ERR_UNSUPPORTED and b["selftest_status"] == kda.KDA_OK
    # no access of the workloads left its buffer
    assert a["status"] == kda.KDA_OK and b["status"] == kda.KDA_OK
    ra, rb = torch.load(tmp_path / "checked.pt"), torch.load(tmp_path / "normal.pt")
    for name in rb:
        for x, y in zip(ra[name], rb[name]):
            assert torch.equal(x, y), name


def test_normal_build_has_no_bounds_self_test(cuda_device):
    if os.path.basename(kda.LIB_PATH) != "libkda.so":
        pytest.skip("the suite runs on another build of the library")
    buf = torch.zeros(16, dtype=torch.uint8, device=cuda_device)
    assert kda.lib().kda_selftest_bounds(buf.data_ptr(), 16, None) == kda.KDA_ERR_UNSUPPORTED
