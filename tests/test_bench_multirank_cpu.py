"""The benchmark's multi-rank plumbing on CPU: two gloo ranks agree on the slowest rank's time and
on the whole-job (weak-scaling) rate, the way `bench.py --gpus N` aggregates its timings."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [12.5, 20.0][rank]
        worst = bench.max_over_ranks(my_ms, world, torch.device("cpu"))
        rate = bench.whole_job_rate(8192.0, world, worst)
        bench.barrier(world)
        out[rank] = (worst, rate)
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_max_time_and_rate():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:  # no fork of this multi-threaded process
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    worst, rate = res[0]
    assert worst == 20.0
    assert rate == pytest.approx(2 * 8192.0 / 0.020)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(100.0, 1, 1000.0) == pytest.approx(100.0)


def test_captured_traffic_follows_the_kernel_sources(tmp_path):
    """The roofline's DRAM traffic comes from the committed ncu capture only while the kernel's
    sources hash to the value recorded with it; any other hash (or workload) gives None."""
    import json

    import bench

    real = bench.kernel_source_hash("chunk_local_tc")
    assert real and bench.kernel_source_hash("no_such_kernel") is None
    assert bench.kernel_source_hash("chunk_state_tc") == real  # one source list for both kernels
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"records": {"chunk_local_tc@w": {"dram_bytes_per_launch": 123,
                                            "source_sha256": real}}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    path = str(prof / "traffic.json")
    assert bench.captured_traffic("chunk_local_tc", "w", path) == 123
    assert bench.captured_traffic("chunk_local_tc", "other", path) is None
    assert bench.captured_traffic("chunk_state_tc", "w", path) is None
    rec["records"]["chunk_local_tc@w"]["source_sha256"] = "0" * 64
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.captured_traffic("chunk_local_tc", "w", path) is None


def test_reference_arm_line_follows_the_contract():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON line with
    the headline keys, our arm's config object, a cpu_baseline describing the run and an e2e
    equal to its own value with no host-device bytes."""
    import json
    import subprocess
    import sys

    import kda_synth

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    run = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], cwd=root, capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stderr[-2000:]
    line = json.loads(run.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 1 and line["value"] > 0
    assert line["config"] == bench.workload_config(kda_synth.STANDARD, 1)
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1


def test_roofline_byte_accounting_matches_the_layouts():
    """The bench's algorithmic bytes, counted by hand from the tensor layouts of the standard
    prefill (B=2, T=4096, H=32, d=128, bf16, C=64: 4096 (chunk, head) items) and the decode. Each
    kernel's share is its part of the method's minimum (inputs to the chunk-local kernel, o and
    the states to the state kernel); the shares add up to the path's minimum, and the records
    between the kernels count for neither."""
    import kda_synth
    from gated_delta_rule_120_b200 import roofline

    spec = kda_synth.STANDARD
    th = 2 * 4096 * 32
    items = 2 * 4096 // 64 * 32
    per_item_inputs = 3 * 64 * 128 * 2 + 64 * 128 * 4 + 64 * 4  # q, k, v bf16; log alpha; beta
    assert per_item_inputs == 82_176
    dims = (th, 2, 32, 128, 128, 2, True, True)
    k1 = roofline.prefill_kernel_share_bytes("chunk_local_tc", *dims)
    assert k1 == items * per_item_inputs
    o_bytes = 2 * 4096 * 32 * 128 * 2
    state = 2 * 32 * 128 * 128 * 4
    k2 = roofline.prefill_kernel_share_bytes("chunk_state_tc", *dims)
    assert k2 == o_bytes + 2 * state  # o written, initial state read, final state written
    # the path's minimum: 1540 B per token-head plus the two states = the two shares
    assert roofline.prefill_min_bytes(*dims) == th * 1540 + 2 * state == k1 + k2
    assert roofline.prefill_kernel_share_bytes("something_else", *dims) is None
    # the roofline block of a step: path frac from the path bytes, kernel fracs from the shares
    prof = [{"name": "chunk_local_tc", "launches": 4, "total_ms": 0.8},
            {"name": "chunk_state_tc", "launches": 4, "total_ms": 0.4}]
    roof = bench.prefill_roofline(spec, 0.3, prof, 4, 6543.4, "measured")
    assert roof["algorithmic_bytes"] == k1 + k2
    assert roof["achieved"] == pytest.approx((k1 + k2) / 0.3e-3 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6543.4)
    assert roof["dominant_kernel"] == "chunk_local_tc"
    kk = {k["name"]: k for k in roof["kernels"]}
    assert kk["chunk_local_tc"]["achieved_gbs"] == pytest.approx(k1 / 0.2e-3 / 1e9)
    assert kk["chunk_state_tc"]["share"] == pytest.approx(1 / 3)
    # decode: every state read once and written once
    assert roofline.decode_state_bytes(256, 32, 128, 128) == 2 * 256 * 32 * 128 * 128 * 4


def test_prefill_path_figures():
    """The path-level figures of the standard prefill at a given step time: minimum bytes, the
    three FLOP-count rates (Eq. 13 < triangular < issued tiles), both tensor-core fractions and
    the roofline-floor fraction; the values of a recorded bench line are reproduced."""
    import kda_synth

    spec = kda_synth.STANDARD
    p = bench.prefill_path_figures(spec, 0.2712591886520386, 6543.4, 1623.7)
    assert p["min_bytes"] == 412_090_368
    assert p["eq13_flops"] == 520_093_696 * 2 * 32
    assert p["eq13_tflops"] == pytest.approx(122.70919451395272, rel=1e-12)
    assert p["frac_tc_peak_eq13"] == pytest.approx(0.07557380951773894, rel=1e-12)
    assert p["frac_tc_datasheet_eq13"] == pytest.approx(p["eq13_tflops"] / 2250.0)
    assert p["eq13_tflops"] < p["triangular_tflops"] < p["issued_tile_tflops"]
    floor_ms = 1e3 * max(412_090_368 / 6543.4e9, p["eq13_flops"] / 1623.7e12)
    assert p["roofline_floor_ms"] == pytest.approx(floor_ms)
    assert p["frac_min_roofline"] == pytest.approx(floor_ms / 0.2712591886520386)
