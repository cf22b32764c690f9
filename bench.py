#!/usr/bin/env python
"""Benchmark of the KDA operator on B200 — prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one chunkwise prefill (kda_chunk_fwd) of the standard prefill batch: B=2, T=4096, H=32,
d_k = d_v = 128, C = 64, bf16 q/k/v, fp32 gates and states, initial state ~ N(0, 0.02^2).
``value`` is prefill tokens/s over all ranks (each rank runs its own batch: weak scaling), with
inputs resident in HBM; ``e2e`` is the same metric through the public API with pinned host
inputs copied in and the outputs read back inside the timed region. Inputs rotate over four
independently drawn sets (> 370 MB, above the 126 MB L2), so no step re-reads a cached input.

Beside it the line carries the decode half of the metric (kda_recurrent_step on 256 sequences x
32 heads with 128 x 128 fp32 states, 1024 steps, state GB/s), the long prefill (B=1, T=131072),
the roofline of the dominant kernel (per-kernel CUDA-event times from the library's profiling
hook), the SM clocks sampled during the timed region, and the fp64 CPU oracle timed on the
host's cores as a reported baseline.

``--impl reference`` times the fp64 CPU oracle (the only reference implementation there is) on a
bounded sample of the same workload per step and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s + % bf16 TC peak (H=32,d=128); decode state GB/s vs HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--decode-steps", type=int, default=1024)
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-long", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[4:8]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        top = max(sm)
        loaded = [x for x in sm if x >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------------- helpers
def dist_setup():
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    """The slowest rank's time (every rank gets it). Works with NCCL (cuda `dev`) and gloo (cpu)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Weak scaling: every rank processes `units_per_rank`; the job's rate is all units over the
    slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


def timed(fn, steps, warmup, world, dev, join=None):
    """W untimed warm-up steps, then K steps between a barrier + synchronize on both sides;
    device time from CUDA events on the launching stream, max over ranks. `join` (optional) makes
    the launching stream wait for work that `fn` queued on other streams before the end event."""
    import torch

    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(steps):
        fn(warmup + i)
    if join is not None:
        join()
    e1.record(s)
    torch.cuda.synchronize(dev)
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


# The files each captured kernel is compiled from: its own source and the headers that source
# includes (the library is one translation unit, but a kernel's code depends only on these).
_TC_SOURCES = ["csrc/kda_chunk_tc.cu", "csrc/kda_common.cuh", "csrc/kda_sm100.cuh",
               "csrc/kda_internal.h", "../include/kda.h"]
KERNEL_SOURCES = {"chunk_local_tc": _TC_SOURCES, "chunk_state_tc": _TC_SOURCES}


def kernel_source_hash(kernel: str) -> str | None:
    """sha256 over the paths and contents of the files `kernel` is compiled from, or None for a
    kernel without a source list."""
    import hashlib

    from gated_delta_rule_120_b200 import _build

    files = KERNEL_SOURCES.get(kernel)
    if files is None:
        return None
    h = hashlib.sha256()
    for rel in files:
        p = os.path.normpath(os.path.join(_build.PKG, rel))
        h.update(os.path.relpath(p, _build.ROOT).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured_traffic(kernel: str, workload: str, path: str | None = None):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu captures
    (profiles/traffic.json, records keyed "kernel@workload"), or None when there is none or the
    kernel's sources changed since it was taken."""
    if path is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                            "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get("records", {}).get(f"{kernel}@{workload}")
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    digest = kernel_source_hash(kernel)
    return rec["dram_bytes_per_launch"] if digest and rec.get("source_sha256") == digest else None


def profile_pass(fn, steps, dev):
    import torch

    import gated_delta_rule_120_b200 as kda

    kda.kda_profile_read()  # drop stale records
    kda.kda_profile_enable(True)
    for i in range(steps):
        fn(i)
    torch.cuda.synchronize(dev)
    kda.kda_profile_enable(False)
    return kda.kda_profile_read()


def chunk_count(spec):
    C = spec.chunk
    if spec.seqlens is None:
        return spec.B * ((spec.T + C - 1) // C)
    return sum((n + C - 1) // C for n in spec.seqlens)


# ---------------------------------------------------------------------------------- arms
def run_prefill(spec, seeds, dev, steps, warmup, world):
    import torch

    import gated_delta_rule_120_b200 as kda
    import kda_synth

    sets = [kda_synth.prefill_inputs(spec, s, dev) for s in seeds]
    o = torch.empty_like(sets[0]["v"])
    fs = torch.empty((spec.num_seqs, spec.H, spec.Dk, spec.Dv), dtype=torch.float32, device=dev)
    ws_bytes = kda.kda_chunk_fwd_workspace_size(spec.B, spec.T, spec.H, spec.Dk, spec.Dv,
                                                spec.chunk, spec.num_seqs, sets[0]["q"].dtype)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step(i):
        x = sets[i % len(sets)]
        kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                          initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                          chunk=spec.chunk, o=o, final_state=fs, workspace=ws)

    ms = timed(step, steps, warmup, world, dev)
    if kda.kda_last_device_error(dev) != kda.KDA_OK:
        raise RuntimeError("device status word set during the prefill benchmark")
    prof = profile_pass(step, steps, dev)
    return dict(ms=ms, prof=prof, sets=sets, o=o, fs=fs, ws=ws, ws_bytes=ws_bytes, step=step)


def run_prefill_e2e(spec, x, o, fs, ws, dev, steps, warmup, world):
    """Public-API end to end: every step copies its inputs from pinned host memory to the device,
    runs kda_chunk_fwd and copies o and the final state back to pinned host memory. Steps are
    pipelined as a serving loop would: host->device copies on one stream, the operator on the
    launching stream, device->host copies on a third, two buffer sets, events between them."""
    import torch

    import gated_delta_rule_120_b200 as kda

    names = ["q", "k", "v", "log_alpha", "beta"] + \
        (["initial_state"] if x["initial_state"] is not None else [])
    host = {n: x[n].cpu().pin_memory() for n in names}
    dbuf = [{n: torch.empty_like(x[n]) for n in names} for _ in range(2)]
    obuf = [(o, fs), (torch.empty_like(o), torch.empty_like(fs))]
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hs = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = ho.numel() * ho.element_size() + hs.numel() * hs.element_size()
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free = [ev(), ev()], [ev(), ev()]
    computed, out_free = [ev(), ev()], [ev(), ev()]
    last_out = [None]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(in_free[b])
            for n in names:
                dbuf[b][n].copy_(host[n], non_blocking=True)
            in_ready[b].record(s_in)
        comp.wait_event(in_ready[b])
        if i >= 2:
            comp.wait_event(out_free[b])
        d, (ob, fb) = dbuf[b], obuf[b]
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                          initial_state=d.get("initial_state"), chunk=spec.chunk, o=ob,
                          final_state=fb, workspace=ws)
        in_free[b].record(comp)
        computed[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            ho.copy_(ob, non_blocking=True)
            hs.copy_(fb, non_blocking=True)
            out_free[b].record(s_out)
        last_out[0] = out_free[b]

    def join():
        comp.wait_event(last_out[0])

    ms = timed(step, steps, warmup, world, dev, join=join)
    torch.cuda.synchronize(dev)
    return ms, h2d, d2h


def run_decode(spec, n_steps, dev, warmup, world, rank, fused=False):
    """Decode steps over the pre-staged inputs of every step; with ``fused`` each step also runs
    the layer's prologue (q/k L2 norm, decay gate from the raw gate) and output epilogue."""
    import torch

    import gated_delta_rule_120_b200 as kda
    import kda_synth

    state = kda_synth.decode_state(spec, 2004 + 10 * rank, dev)
    x = kda_synth.decode_step_inputs(spec, 2004 + 10 * rank, n_steps, dev)
    o = torch.empty((spec.N, spec.H, spec.Dv), dtype=x["q"].dtype, device=dev)
    fusion = None
    if fused:
        g = torch.Generator(device=dev).manual_seed(2104 + 10 * rank)
        fusion = dict(qk_l2norm=True, eps=1e-6,
                      A_log=torch.log(torch.rand((spec.H,), generator=g, device=dev) * 15 + 1) - 2,
                      dt_bias=torch.randn((spec.H, spec.Dk), generator=g, device=dev) * 0.5,
                      out_norm=True, out_norm_eps=1e-5,
                      out_norm_weight=torch.rand((spec.Dv,), generator=g, device=dev) + 0.5,
                      out_gate=torch.randn(o.shape, generator=g, device=dev).to(o.dtype))

    def step(i):
        s = i % n_steps
        kda.kda_recurrent_step(x["q"][s], x["k"][s], x["v"][s], x["log_alpha"][s], x["beta"][s],
                               state, o=o, fusion=fusion)

    ms = timed(step, n_steps, warmup, world, dev)
    prof = profile_pass(step, min(n_steps, 64), dev)
    del x
    return ms, prof


def run_fused_prefill(spec, seed, dev, steps, warmup, world, epilogue=False):
    """Standard prefill through kda_chunk_fwd with the fused prologue: raw (un-normalised) q, k and
    raw decay gates turned into log decays in-kernel from A_log and dt_bias; with ``epilogue`` the
    output is also normalised head-wise and gated (RMSNorm x sigmoid) before the store."""
    import torch

    import gated_delta_rule_120_b200 as kda
    import kda_synth

    x = kda_synth.prefill_inputs(spec, seed, dev)
    g = torch.Generator(device=dev).manual_seed(seed + 7)
    q = (x["q"].float() * 3.0).to(x["q"].dtype)
    k = (x["k"].float() * 3.0).to(x["k"].dtype)
    gate = torch.randn(x["log_alpha"].shape, generator=g, device=dev) - 1.0
    fusion = dict(qk_l2norm=True, eps=1e-6,
                  A_log=torch.log(torch.rand((spec.H,), generator=g, device=dev) * 15 + 1) - 2.0,
                  dt_bias=torch.randn((spec.H, spec.Dk), generator=g, device=dev) * 0.5)
    if epilogue:
        fusion.update(out_norm=True, out_norm_eps=1e-5,
                      out_norm_weight=torch.rand((spec.Dv,), generator=g, device=dev) + 0.5,
                      out_gate=torch.randn(x["v"].shape, generator=g, device=dev).to(x["v"].dtype))
    o = torch.empty_like(x["v"])
    fs = torch.empty((spec.num_seqs, spec.H, spec.Dk, spec.Dv), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_size(spec.B, spec.T, spec.H, spec.Dk, spec.Dv,
                                                      spec.chunk, spec.num_seqs, q.dtype),
                     dtype=torch.uint8, device=dev)

    def step(i):
        kda.kda_chunk_fwd(q, k, x["v"], gate, x["beta"], initial_state=x["initial_state"],
                          chunk=spec.chunk, o=o, final_state=fs, workspace=ws, fusion=fusion)

    return timed(step, steps, warmup, world, dev)


def run_recurrent_mode(N, T, H, D, dev, steps, warmup, world, seed, fused=False):
    """Multi-token recurrent mode (kda_recurrent_fwd): N sequences x T tokens applied to states
    gathered from a pool by index (serving-cache layout); bf16 q/k/v, fp32 gates and states. With
    ``fused`` the layer's prologue and epilogue run in the kernel: raw q/k L2-normalised, the log
    decay formed from a raw gate (A_log, dt_bias), the output RMS-normalised, weighted and gated."""
    import torch

    import gated_delta_rule_120_b200 as kda
    import kda_synth

    spec = kda_synth.PrefillSpec("recurrent", B=N, T=T, H=H, Dk=D, Dv=D, chunk=64, dtype="bf16",
                                 decay="slow", init_std=0.0)
    x = kda_synth.prefill_inputs(spec, seed, dev)
    g = torch.Generator(device=dev).manual_seed(seed + 1)
    P = 2 * N
    pool = torch.randn((P, H, D, D), generator=g, device=dev) * 0.02
    idx = torch.randperm(P, generator=g, device=dev)[:N].to(torch.int32)
    o = torch.empty_like(x["v"])
    fusion = None
    if fused:
        x["q"] = (x["q"].float() * 3.0).to(x["q"].dtype)
        x["k"] = (x["k"].float() * 3.0).to(x["k"].dtype)
        x["log_alpha"] = torch.randn(x["log_alpha"].shape, generator=g, device=dev) - 1.0
        fusion = dict(qk_l2norm=True, eps=1e-6,
                      A_log=torch.log(torch.rand((H,), generator=g, device=dev) * 15 + 1) - 2.0,
                      dt_bias=torch.randn((H, D), generator=g, device=dev) * 0.5,
                      out_norm=True, out_norm_eps=1e-5,
                      out_norm_weight=torch.rand((D,), generator=g, device=dev) + 0.5,
                      out_gate=torch.randn(x["v"].shape, generator=g, device=dev).to(x["v"].dtype))

    def step(i):
        kda.kda_recurrent_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, idx, o=o,
                              fusion=fusion)

    return timed(step, steps, warmup, world, dev)


def run_backward(spec, seed, dev, steps, warmup, world):
    """The backward pass (kda_chunk_bwd) of the standard prefill: gradients of every input for a
    random output cotangent and final-state cotangent. Returns (ms over `steps`, profile)."""
    import torch

    import gated_delta_rule_120_b200 as kda
    import kda_synth

    x = kda_synth.prefill_inputs(spec, seed, dev)
    g = torch.Generator(device=dev).manual_seed(seed + 3)
    d_o = torch.randn(x["v"].shape, generator=g, device=dev).to(x["v"].dtype)
    d_fin = torch.randn((spec.num_seqs, spec.H, spec.Dk, spec.Dv), generator=g, device=dev)
    ws = torch.empty(kda.kda_chunk_bwd_workspace_size(spec.B, spec.T, spec.H, spec.Dk, spec.Dv,
                                                      spec.num_seqs, x["q"].dtype),
                     dtype=torch.uint8, device=dev)

    def step(i):
        kda.kda_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                          initial_state=x["initial_state"], d_final_state=d_fin, workspace=ws)

    ms = timed(step, steps, warmup, world, dev)
    prof = profile_pass(step, 2, dev)
    return ms, prof


def cpu_baseline(spec, dev, budget_s):
    """The fp64 oracle as it stands, on the host's cores, over whole sequences of the prefill
    workload (all heads), repeated until ~budget_s of CPU work. Returns tokens/s."""
    import kda_synth
    import oracle

    x = kda_synth.prefill_inputs(spec, 2001, "cpu")
    done, t0 = 0, time.perf_counter()
    n = 0
    while True:
        b = n % spec.B
        s0 = None if x["initial_state"] is None else x["initial_state"][b:b + 1]
        oracle.recurrent(x["q"][b], x["k"][b], x["v"][b], x["log_alpha"][b], x["beta"][b],
                         initial_state=s0)
        done += spec.T
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return dict(value=done / el, unit="tokens/s", cores=oracle.max_threads(), kind="oracle",
                sample=f"{n} whole sequences of {spec.T} tokens x {spec.H} heads (fp64 "
                       f"token-by-token recurrence, OpenMP over heads), {el:.1f} s")


def prefill_roofline(spec, ms_step: float, prof, steps: int, hbm_peak: float,
                     peak_src: str) -> dict:
    """Roofline of one prefill call (the path: every kernel of kda_chunk_fwd) against the method's
    algorithmic bytes (per token-head q, k, v, o in the input dtype, log_alpha fp32, beta fp32;
    the fp32 states in and out), with each kernel's share of those bytes beside its own CUDA-event
    time. `traffic` is the DRAM bytes the path's kernels really moved, from the committed ncu
    captures (None while any is missing or stale); its ratio to the algorithmic bytes shows the
    cost of the records the chunk-local kernel writes and the state kernel reads."""
    from gated_delta_rule_120_b200 import roofline

    qkv = 2 if spec.dtype == "bf16" else 4
    th = spec.token_heads()
    dims = (th, spec.num_seqs, spec.H, spec.Dk, spec.Dv, qkv, spec.init_std > 0, True)
    alg = roofline.prefill_min_bytes(*dims)
    total = sum(p["total_ms"] for p in prof) or 1.0
    kernels, traffic, complete = [], 0.0, True
    for p in sorted(prof, key=lambda p: -p["total_ms"]):
        ms = p["total_ms"] / p["launches"]
        share = roofline.prefill_kernel_share_bytes(p["name"], *dims)
        tr = captured_traffic(p["name"], spec.name)
        per_step = p["launches"] / steps
        kernels.append({
            "name": p["name"], "launches_per_step": per_step, "ms_per_launch": ms,
            "share": p["total_ms"] / total, "algorithmic_bytes": share,
            "achieved_gbs": share / (ms / 1e3) / 1e9 if share else None,
            "frac": share / (ms / 1e3) / 1e9 / hbm_peak if share else None,
            "traffic": tr, "traffic_over_algorithmic": tr / share if tr and share else None})
        if tr is None:
            complete = False
        else:
            traffic += tr * per_step
    achieved = alg / (ms_step / 1e3) / 1e9
    return {"kernel": "kda_chunk_fwd (" + " + ".join(k["name"] for k in kernels) + ")",
            "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "traffic": traffic if complete else None,
            "traffic_over_algorithmic": traffic / alg if complete else None,
            "algorithmic_bytes": alg,
            "algorithmic_basis": "per token-head q, k, v, o in the input dtype + log_alpha fp32 + "
                                 "beta fp32 (1540 B at d = 128, bf16) + fp32 states in and out",
            "peak_source": f"{peak_src} HBM copy bandwidth", "launch_ms": ms_step,
            "dominant_kernel": kernels[0]["name"] if kernels else None, "kernels": kernels}


DATASHEET_BF16_TFLOPS = 2250.0  # nominal dense bf16 tensor-core peak of one B200


def prefill_path_figures(spec, ms_step: float, hbm_peak: float, tc_peak: float) -> dict:
    """Path-level figures of one prefill step of `spec` taking `ms_step` ms: minimum HBM bytes and
    their rate, the three FLOP counts (Eq. 13, triangular halves excluded, full issued tiles) as
    rates, Eq. 13 as a fraction of the measured and of the datasheet tensor-core peak, and the
    fraction of the min(TC, HBM) roofline floor. Peaks in GB/s and TFLOP/s."""
    from gated_delta_rule_120_b200 import roofline

    sec = ms_step / 1e3
    heads = spec.B * spec.H
    min_bytes = roofline.prefill_min_bytes(spec.token_heads(), spec.num_seqs, spec.H, spec.Dk,
                                           spec.Dv, 2, spec.init_std > 0, True)
    eq13 = roofline.eq13_flops(spec.T, spec.chunk, spec.Dk) * heads
    path = {"min_bytes": min_bytes, "achieved_gbs": min_bytes / sec / 1e9,
            "frac_hbm": min_bytes / sec / 1e9 / hbm_peak,
            "eq13_flops": eq13, "eq13_tflops": eq13 / sec / 1e12,
            "frac_tc_peak_eq13": eq13 / sec / 1e12 / tc_peak,
            "frac_tc_datasheet_eq13": eq13 / sec / 1e12 / DATASHEET_BF16_TFLOPS,
            "triangular_tflops": roofline.triangular_flops(spec.T, spec.chunk, spec.Dk) *
            heads / sec / 1e12,
            "issued_tile_tflops": roofline.issued_tile_flops(spec.T, spec.chunk, spec.Dk) *
            heads / sec / 1e12,
            "roofline_floor_ms": 1e3 * max(min_bytes / (hbm_peak * 1e9),
                                           eq13 / (tc_peak * 1e12))}
    path["frac_min_roofline"] = path["roofline_floor_ms"] / ms_step
    return path


def workload_config(spec, world: int) -> dict:
    """The `config` object of the headline line, the same for both arms."""
    return {"workload": spec.name, "B": spec.B, "T": spec.T, "H": spec.H,
            "d_k": spec.Dk, "d_v": spec.Dv, "chunk": spec.chunk,
            "state": "fp32", "gates": "fp32",
            "l2": "4 rotating input sets (>370 MB) larger than the 126 MB L2",
            "parallelism": f"dp{world} (independent batches per GPU)"}


def reference_arm(args, world, rank):
    """--impl reference: the fp64 CPU oracle on a bounded sample of the same workload per step."""
    if rank != 0:
        return
    import kda_synth
    import oracle

    spec = kda_synth.STANDARD
    x = kda_synth.prefill_inputs(spec, 2001, "cpu")
    heads = 8  # per step: one sequence, 8 of the 32 heads, all 4096 tokens
    sub = {n: x[n][0, :, :heads].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    s0 = x["initial_state"][0:1, :heads].contiguous()

    def step():
        oracle.recurrent(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                         initial_state=s0)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    tokens_per_s = args.steps * spec.T * heads / spec.H / el  # whole-head-equivalent tokens
    line = {
        "impl": "reference", "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(spec, args.gpus),
        "cpu_baseline": {"value": tokens_per_s, "unit": "tokens/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"per step: 1 sequence x {heads} of {spec.H} heads x "
                                   f"{spec.T} tokens, scaled to whole-head tokens"},
        "e2e": {"value": tokens_per_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return

    import torch

    import gated_delta_rule_120_b200 as kda
    import kda_synth
    from gated_delta_rule_120_b200 import roofline

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.lib()
    peaks, peak_src = load_peaks()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"

    spec = kda_synth.STANDARD
    seeds = [2001 + 10 * rank + r for r in range(4)]
    with ClockSampler(uuid if rank == 0 else None) as clk:
        pre = run_prefill(spec, seeds, dev, args.steps, args.warmup, world)
    clocks = clk.summary() if rank == 0 else None
    ms_step = pre["ms"] / args.steps
    tokens = spec.total_tokens
    value = whole_job_rate(tokens * args.steps, world, pre["ms"])

    # roofline of the prefill path, with each kernel's share of the algorithmic bytes
    prof = pre["prof"]
    launches_per_step = sum(p["launches"] for p in prof) / args.steps
    hbm_peak = peaks["hbm_gbs"]
    roof = prefill_roofline(spec, ms_step, prof, args.steps, hbm_peak, peak_src)
    # path-level figures for the prefill step
    path = prefill_path_figures(spec, ms_step, hbm_peak, peaks["bf16_tflops"])

    # public-API end to end
    e2e_ms, h2d, d2h = run_prefill_e2e(spec, pre["sets"][0], pre["o"], pre["fs"], pre["ws"], dev,
                                       args.steps, args.warmup, world)
    e2e = {"value": world * tokens * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms / args.steps}
    del pre
    torch.cuda.empty_cache()

    extra = {}
    if not args.no_long:
        lspec = kda_synth.LONG
        lsteps = max(2, args.steps // 5)
        lp = run_prefill(lspec, [2002 + 10 * rank], dev, lsteps, 1, world)
        lms = lp["ms"] / lsteps
        lpath = prefill_path_figures(lspec, lms, hbm_peak, peaks["bf16_tflops"])
        extra["long_prefill"] = {
            "workload": lspec.name, "tokens_per_s": world * lspec.total_tokens / (lms / 1e3),
            "ms_per_call": lms, "frac_hbm_min_bytes": lpath["frac_hbm"],
            "eq13_tflops": lpath["eq13_tflops"],
            "roofline": prefill_roofline(lspec, lms, lp["prof"], lsteps, hbm_peak, peak_src),
            "prefill_path": lpath}
        del lp
        torch.cuda.empty_cache()
        # packed variable-length batch: 16 sequences, lengths log-uniform in [256, 32768]
        vspec = kda_synth.varlen_spec(1003)
        vsteps = max(2, args.steps // 5)
        vp = run_prefill(vspec, [2003 + 10 * rank], dev, vsteps, 2, world)
        vms = vp["ms"] / vsteps
        vmin = roofline.prefill_min_bytes(vspec.token_heads(), vspec.num_seqs, vspec.H, vspec.Dk,
                                          vspec.Dv, 2, False, True)
        veq13 = sum(roofline.eq13_flops(n_tok, 64, 128) for n_tok in vspec.seqlens) * vspec.H
        extra["varlen_prefill"] = {
            "workload": vspec.name, "sequences": vspec.num_seqs,
            "tokens": vspec.total_tokens, "longest": max(vspec.seqlens),
            "tokens_per_s": world * vspec.total_tokens / (vms / 1e3),
            "ms_per_call": vms, "frac_hbm_min_bytes": vmin / (vms / 1e3) / 1e9 / hbm_peak,
            "eq13_tflops": veq13 / (vms / 1e3) / 1e12,
            "kernels": [{"name": p["name"], "ms_per_launch": p["total_ms"] / p["launches"]}
                        for p in vp["prof"]]}
        del vp
        torch.cuda.empty_cache()
    # the fused prologue on the standard workload
    fms = run_fused_prefill(spec, 2001 + 10 * rank, dev, args.steps, args.warmup, world)
    extra["fused_prologue_prefill"] = {
        "workload": spec.name + "_raw_qk_and_gates",
        "tokens_per_s": whole_job_rate(tokens * args.steps, world, fms),
        "ms_per_call": fms / args.steps,
        "overhead_vs_plain": (fms / args.steps) / ms_step - 1.0}
    # prologue + output epilogue (head-wise RMSNorm x sigmoid gate fused into the state kernel)
    lms = run_fused_prefill(spec, 2001 + 10 * rank, dev, args.steps, args.warmup, world,
                            epilogue=True)
    extra["fused_layer_prefill"] = {
        "workload": spec.name + "_raw_qk_gates_and_output_gate",
        "tokens_per_s": whole_job_rate(tokens * args.steps, world, lms),
        "ms_per_call": lms / args.steps,
        "overhead_vs_plain": (lms / args.steps) / ms_step - 1.0}
    # the multi-token recurrent mode: 256 sequences x 16 tokens x 32 heads, states from a pool
    rN, rT = 256, 16
    rsteps = max(3, args.steps // 2)
    rms = run_recurrent_mode(rN, rT, 32, 128, dev, rsteps, 2, world, 2005 + 10 * rank)
    per = rms / rsteps
    rstate = roofline.decode_state_bytes(rN, 32, 128, 128)
    rtotal = rstate + rN * 32 * rT * ((3 * 128) * 2 + 4 * 128 + 4 + 128 * 2)
    extra["recurrent_mode"] = {
        "workload": f"recurrent_N{rN}_T{rT}_H32_d128_pool",
        "tokens_per_s": whole_job_rate(rN * rT, world, per),
        "ms_per_call": per,
        "achieved_gbs": rtotal / (per / 1e3) / 1e9,
        "frac_hbm": rtotal / (per / 1e3) / 1e9 / hbm_peak}
    fms = run_recurrent_mode(rN, rT, 32, 128, dev, rsteps, 2, world, 2015 + 10 * rank, fused=True)
    fper = fms / rsteps
    ftotal = rtotal + rN * 32 * rT * 128 * 2  # + the output-gate rows
    extra["recurrent_mode"]["fused"] = {
        "workload": f"recurrent_N{rN}_T{rT}_H32_d128_pool_fused_prologue_epilogue",
        "tokens_per_s": whole_job_rate(rN * rT, world, fper),
        "ms_per_call": fper,
        "achieved_gbs": ftotal / (fper / 1e3) / 1e9,
        "frac_hbm": ftotal / (fper / 1e3) / 1e9 / hbm_peak}
    torch.cuda.empty_cache()
    # the backward pass of the standard prefill
    bsteps = max(3, args.steps // 4)
    bms, bprof = run_backward(spec, 2007 + 10 * rank, dev, bsteps, 2, world)
    extra["backward"] = {
        "workload": spec.name + "_backward",
        "tokens_per_s": whole_job_rate(tokens * bsteps, world, bms),
        "ms_per_call": bms / bsteps,
        "vs_forward": (bms / bsteps) / ms_step,
        "kernels": [{"name": p["name"], "ms_per_launch": p["total_ms"] / p["launches"]}
                    for p in bprof]}
    torch.cuda.empty_cache()
    if not args.no_decode:
        dspec = kda_synth.DECODE
        dms, dprof = run_decode(dspec, args.decode_steps, dev, 3, world, rank)
        sbytes = roofline.decode_state_bytes(dspec.N, dspec.H, dspec.Dk, dspec.Dv)
        tbytes = roofline.decode_total_bytes(dspec.N, dspec.H, dspec.Dk, dspec.Dv, 2)
        per = dms / args.decode_steps
        kms = dprof[0]["total_ms"] / dprof[0]["launches"]
        # the same decode steps with the layer's prologue and output epilogue fused in
        fsteps = args.decode_steps  # as many steps as the plain run, so the two compare
        fdms, _ = run_decode(dspec, fsteps, dev, 3, world, rank, fused=True)
        fper = fdms / fsteps
        fused_decode = {"workload": dspec.name + "_fused_prologue_epilogue", "steps": fsteps,
                        "ms_per_step": fper,
                        "state_gbs": world * sbytes / (fper / 1e3) / 1e9,
                        "frac_hbm_state": sbytes / (fper / 1e3) / 1e9 / hbm_peak}
        extra["decode"] = {
            "workload": dspec.name, "steps": args.decode_steps, "ms_per_step": per,
            "state_gbs": world * sbytes / (per / 1e3) / 1e9,
            "frac_hbm_state": sbytes / (per / 1e3) / 1e9 / hbm_peak,
            "total_gbs": world * tbytes / (per / 1e3) / 1e9,
            "kernel": {"name": dprof[0]["name"], "ms_per_launch": kms,
                       "achieved_gbs": tbytes / (kms / 1e3) / 1e9,
                       "frac": tbytes / (kms / 1e3) / 1e9 / hbm_peak},
            "fused": fused_decode}
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, dev, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(spec, world),
            "roofline": roof, "prefill_path": path, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "clocks": clocks, **extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
